// Device kernels for layerwise QK-RMSNorm on sm_100a.
//
// Method: "SwiftQK: Fast and Communication-Efficient Tensor Parallelism for
// Query-Key Normalization" (arXiv 2608.09160).
//   Background, RMS-Norm (Equation 1): r = 1 / sqrt(sum_j x_j^2 / H + eps),
//     y_j = x_j * gamma_j * r, per full projected Q row and K row.
//   Phase A: per-shard squared sums, added in fp32, give the global sum.
//   Phase B: x * gamma does not depend on the reduction; r scales it on the
//     way out and only the final values are written.
//   Deadlock-safe persistent execution: a bounded grid of resident CTAs that
//     loop over tokens (here: over the Q rows, then the K rows).
//   Evaluation, Fig. 2(b): BF16 and FP8-E4M3 activations with FP32
//     accumulation.
//
// The work is a read-once / write-once stream with a per-row reduction: no
// contraction, so no tensor cores.  What matters on B200 is bytes in flight
// per SM (16-byte coalesced vectors, several rows per SM outstanding), a short
// per-row critical path, and a grid bounded by residency.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {

enum Mode : int {
    kFused = 0,  // sum of squares -> factor -> scale and store
    kStats = 1,  // sum of squares -> write fp32 partial sum
    kApply = 2   // combine P partial sums -> factor -> scale and store
};

// One tensor's rows (Q or K, or a shard of one).  Kept compact (96 bytes):
// every launch copies the row sets as kernel parameters, and the small,
// latency-bound launches (decode, tiny batches) pay for each byte.
struct RowSet {
    const char *in;          // row t starts at in + t * stride_bytes
    char *out;               // kFused / kApply
    const char *gamma;       // kFused / kApply, [width] of the gamma type
    union {
        float *sumsq;            // kStats: [T]
        const float *sumsq_all;  // kApply: [P][T]
    };
    int64_t stride_bytes;
    int64_t head_bytes;      // headwise: bytes from one head to the next within a token's row
    int64_t rows;            // T * heads
    int64_t item_end;        // register kernel: items of this set and of every set before it
    int32_t P;               // kApply: partial sums per token in sumsq_all
    int32_t width;           // elements in this row (shard width for kStats / kApply)
    int32_t nfull;           // full 16-byte vectors of x in the row
    int32_t tail;            // elements after the last full vector
    float inv_div;           // 1 / (the FULL width), rounded to fp32 on the host
    int32_t heads;           // rows per token: 1 (layerwise) or the number of heads (headwise)
    int32_t group;           // register kernel: threads that share one row (1..16, or a multiple of 32)
    int32_t rows_per_item;   // register kernel: blockDim / group rows handled per item
};
static_assert(sizeof(RowSet) == 96, "row set layout");

// The row sets of one launch: Q then K (SETS = 2), or -- for the multi-shard
// forms of Phase A's local step and of the combine/apply -- the P Q shards
// then the P K shards (SETS = kMaxShardSets, nsets = 2P of them in use).
template <int SETS>
struct ParamsT {
    RowSet set[SETS];
    int32_t nsets;           // sets in use
    int64_t n_items;         // register kernel: items over all sets in use
    int64_t T;
    float eps;
};
using Params = ParamsT<2>;   // 0 = Q, 1 = K
constexpr int kMaxShards = 8;
constexpr int kMaxShardSets = 2 * kMaxShards;
using ShardParams = ParamsT<kMaxShardSets>;

// ----------------------------------------------------------------------------
// Packed fp32 pairs.  sm_100 executes add/mul/fma on two fp32 lanes held in
// one 64-bit register pair (PTX .f32x2); each lane is an ordinary IEEE
// round-to-nearest operation, so results equal the scalar ones bit for bit
// while the instruction count of the elementwise work halves.
struct F2 {
    unsigned long long v;
};
__device__ __forceinline__ F2 f2(float lo, float hi) {
    return F2{static_cast<unsigned long long>(__float_as_uint(lo)) |
              (static_cast<unsigned long long>(__float_as_uint(hi)) << 32)};
}
__device__ __forceinline__ F2 f2_bits(uint32_t lo_bits, uint32_t hi_bits) {
    return F2{static_cast<unsigned long long>(lo_bits) | (static_cast<unsigned long long>(hi_bits) << 32)};
}
__device__ __forceinline__ float f2_lo(F2 a) { return __uint_as_float(static_cast<uint32_t>(a.v)); }
__device__ __forceinline__ float f2_hi(F2 a) { return __uint_as_float(static_cast<uint32_t>(a.v >> 32)); }
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
    F2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
    F2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
    return d;
}

// ----------------------------------------------------------------------------
// Element types.  For each: the storage of one element (Bits), elements per
// 16-byte vector (kPerVec), the gamma type (G) and how many 16-byte gamma
// vectors cover the elements of one x vector (kGVecs); conversions of a whole
// vector to / from fp32 pairs, and of one element.  Narrowing rounds to
// nearest even (E4M3: and saturates to +-448, the format having no infinity).
template <typename E>
struct Elem;

template <>
struct Elem<float> {
    using Bits = uint32_t;
    using G = float;
    static constexpr int kPerVec = 4;
    static constexpr int kGVecs = 1;
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[kPerVec / 2]) {
        p[0] = f2_bits(v.x, v.y);
        p[1] = f2_bits(v.z, v.w);
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[kPerVec / 2]) {
        return make_uint4(static_cast<uint32_t>(p[0].v), static_cast<uint32_t>(p[0].v >> 32),
                          static_cast<uint32_t>(p[1].v), static_cast<uint32_t>(p[1].v >> 32));
    }
    __device__ __forceinline__ static float to_float(Bits b) { return __uint_as_float(b); }
    __device__ __forceinline__ static Bits from_float(float f) { return __float_as_uint(f); }
};

template <>
struct Elem<__nv_bfloat16> {
    using Bits = uint16_t;
    using G = __nv_bfloat16;
    static constexpr int kPerVec = 8;
    static constexpr int kGVecs = 1;
    // the bf16 in the low half of a word is the fp32 with those bits in the high half
    __device__ __forceinline__ static F2 widen_word(uint32_t w) { return f2_bits(w << 16, w & 0xFFFF0000u); }
    __device__ __forceinline__ static uint32_t narrow_word(F2 a) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f2_lo(a), f2_hi(a));
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[kPerVec / 2]) {
        p[0] = widen_word(v.x);
        p[1] = widen_word(v.y);
        p[2] = widen_word(v.z);
        p[3] = widen_word(v.w);
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[kPerVec / 2]) {
        return make_uint4(narrow_word(p[0]), narrow_word(p[1]), narrow_word(p[2]), narrow_word(p[3]));
    }
    __device__ __forceinline__ static float to_float(Bits b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
    __device__ __forceinline__ static Bits from_float(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
};

template <>
struct Elem<__half> {
    using Bits = uint16_t;
    using G = __half;
    static constexpr int kPerVec = 8;
    static constexpr int kGVecs = 1;
    __device__ __forceinline__ static F2 widen_word(uint32_t w) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
        return f2(f.x, f.y);
    }
    __device__ __forceinline__ static uint32_t narrow_word(F2 a) {
        __half2 h = __floats2half2_rn(f2_lo(a), f2_hi(a));
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[kPerVec / 2]) {
        p[0] = widen_word(v.x);
        p[1] = widen_word(v.y);
        p[2] = widen_word(v.z);
        p[3] = widen_word(v.w);
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[kPerVec / 2]) {
        return make_uint4(narrow_word(p[0]), narrow_word(p[1]), narrow_word(p[2]), narrow_word(p[3]));
    }
    __device__ __forceinline__ static float to_float(Bits b) { return __half2float(__ushort_as_half(b)); }
    __device__ __forceinline__ static Bits from_float(float f) { return __half_as_ushort(__float2half_rn(f)); }
};

template <>
struct Elem<__nv_fp8_e4m3> {
    using Bits = uint8_t;
    using G = __nv_bfloat16;  // gamma is kept in bf16 next to E4M3 activations
    static constexpr int kPerVec = 16;
    static constexpr int kGVecs = 2;
    // two E4M3 values (16 bits) -> exact half pair -> fp32 pair
    __device__ __forceinline__ static F2 widen_half_word(uint32_t two) {
        const __half2_raw hr =
            __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
        return f2(f.x, f.y);
    }
    __device__ __forceinline__ static uint32_t narrow_pair(F2 a) {
        return static_cast<uint32_t>(
            __nv_cvt_float2_to_fp8x2(make_float2(f2_lo(a), f2_hi(a)), __NV_SATFINITE, __NV_E4M3));
    }
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[kPerVec / 2]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            p[2 * i] = widen_half_word(w[i]);
            p[2 * i + 1] = widen_half_word(w[i] >> 16);
        }
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[kPerVec / 2]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = narrow_pair(p[2 * i]) | (narrow_pair(p[2 * i + 1]) << 16);
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ __forceinline__ static float to_float(Bits b) {
        const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
        return __half2float(*reinterpret_cast<const __half *>(&hr));
    }
    __device__ __forceinline__ static Bits from_float(float f) {
        return static_cast<Bits>(__nv_cvt_float_to_fp8(f, __NV_SATFINITE, __NV_E4M3));
    }
};

// ----------------------------------------------------------------------------
// Memory access.  x is streamed (read once, evict first); it may be the same
// memory as the output (in place), so it is read through the coherent path.
// gamma is never written during a launch (the host rejects any overlap with an
// output) and is shared by every row: read-only path, cached.
__device__ __forceinline__ uint4 ld_stream(const char *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_stream(char *p, const uint4 &v) {
    __stcs(reinterpret_cast<uint4 *>(p), v);
}
__device__ __forceinline__ uint4 ld_gamma(const char *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// The last, partial vector of a row: `n` (< kPerVec) elements, the rest zero.
template <typename E>
__device__ __forceinline__ uint4 ld_tail(const char *p, int n) {
    using B = typename Elem<E>::Bits;
    constexpr int N = Elem<E>::kPerVec;
    B b[N];
    const B *src = reinterpret_cast<const B *>(p);
#pragma unroll
    for (int e = 0; e < N; ++e) b[e] = (e < n) ? src[e] : B(0);
    uint4 v;
    static_assert(sizeof(b) == sizeof(uint4), "vector size");
    memcpy(&v, b, sizeof(v));
    return v;
}
template <typename E>
__device__ __forceinline__ void st_tail(char *p, const uint4 &v, int n) {
    using B = typename Elem<E>::Bits;
    constexpr int N = Elem<E>::kPerVec;
    B b[N];
    memcpy(b, &v, sizeof(v));
    B *dst = reinterpret_cast<B *>(p);
#pragma unroll
    for (int e = 0; e < N; ++e)
        if (e < n) dst[e] = b[e];
}

// The gamma vectors covering x vector `vi` of a row of `nfull` full vectors
// and `tail` trailing elements (zero past the row's end).
template <typename E>
__device__ __forceinline__ void ld_gamma_vec(const char *gamma, int vi, int nfull, int tail,
                                             uint4 (&g)[Elem<E>::kGVecs]) {
    using GB = typename Elem<typename Elem<E>::G>::Bits;
    constexpr int KG = Elem<E>::kGVecs;
    const char *p = gamma + static_cast<int64_t>(vi) * 16 * KG;
    if (vi < nfull) {
#pragma unroll
        for (int j = 0; j < KG; ++j) g[j] = ld_gamma(p + 16 * j);
    } else if (vi == nfull && tail) {
        constexpr int N = Elem<E>::kPerVec;
        GB b[N];
        const GB *src = reinterpret_cast<const GB *>(p);
#pragma unroll
        for (int e = 0; e < N; ++e) b[e] = (e < tail) ? src[e] : GB(0);
        static_assert(sizeof(b) == sizeof(g), "gamma vector size");
        memcpy(g, b, sizeof(b));
    } else {
#pragma unroll
        for (int j = 0; j < KG; ++j) g[j] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ----------------------------------------------------------------------------
// Reductions.  The block sum is formed in a fixed order (warp butterfly, then
// warp partials added 0..nwarps-1 by every thread), so every thread of a CTA
// holds the same value and a run is deterministic.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

// Sum over aligned groups of `g` lanes (g a power of two below 32): butterfly
// with offsets g/2 .. 1 keeps the groups apart.
__device__ __forceinline__ float segment_sum(float v, int g) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        if (off < g) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

// Row r of a tensor -> the byte offset of its first element: token r / heads,
// head r % heads.
__device__ __forceinline__ int64_t row_offset(int64_t r, int heads, int64_t stride, int64_t head_bytes) {
    if (heads == 1) return r * stride;
    const uint32_t rr = static_cast<uint32_t>(r);  // headwise rows are fewer than 2^31 (host check)
    const uint32_t t = rr / static_cast<uint32_t>(heads);
    return static_cast<int64_t>(t) * stride + static_cast<int64_t>(rr - t * heads) * head_bytes;
}

// `red` has two slots of 32 floats; alternating slots between consecutive rows
// lets one barrier per row suffice: a thread can only overwrite slot s after
// every thread has passed the barrier of the row in between, i.e. after all
// reads of slot s are done.
__device__ __forceinline__ float block_sum(float v, float (*red)[32], int &slot) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    v = warp_sum(v);
    if (lane == 0) red[slot][warp] = v;
    __syncthreads();
    float s = 0.0f;
    for (int w = 0; w < nwarps; ++w) s += red[slot][w];
    slot ^= 1;
    return s;
}

// Phase A aggregation: the P partial sums of token t (all[p * T + t]) added
// in order p = 0, 1, ..., P-1 in fp32.  The lanes of a warp that share row t
// split the loads: lane li (< width, a power of two <= 32, the lane's index
// within its row group) loads partials li, li + width, ..., and every lane
// adds all P values in order from shuffles, so each gets the same sequential
// sum with one load instead of P.  Every lane of the warp must call it
// (inactive rows pass active = false and load nothing).
__device__ __forceinline__ float combine_partials_lanes(const float *all, int64_t T, int P, int64_t t, bool active,
                                                        int li, int width) {
    float s = 0.0f;
    for (int p0 = 0; p0 < P; p0 += width) {
        const int q = p0 + li;
        const float v = (active && q < P) ? __ldg(all + static_cast<int64_t>(q) * T + t) : 0.0f;
        const int n = P - p0 < width ? P - p0 : width;
        for (int i = 0; i < n; ++i) s += __shfl_sync(0xFFFFFFFFu, v, i, width);
    }
    return s;
}

// r = 1 / sqrt(S / H + eps), the mean formed as S * fl(1 / H); the product
// and the sum are one fused multiply-add (rounded once).
__device__ __forceinline__ float rms_factor(float sumsq, float inv_div, float eps) {
    return rsqrtf(__fmaf_rn(sumsq, inv_div, eps));
}

// Programmatic dependent launch (sm_90+).  Kernels here are launched with
// programmatic stream serialization, so their CTAs may be dispatched while the
// previous kernel in the stream is still draining.  Every kernel therefore
// first waits until that kernel has completed and its memory operations are
// visible (a no-op when launched without the attribute), and at once allows
// the next kernel to be dispatched as its own CTAs retire; that kernel waits
// for this one's completion in turn.
__device__ __forceinline__ void pdl_wait_and_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Squared sum of a thread's vectors (two fp32 lanes accumulate the even and
// odd elements; they are added at the end).
// Squares of the two halves of an f16x2 word added to the even and odd
// accumulators with sm_100's mixed-precision fma (f16 inputs, fp32 addend and
// result).  An f16 x f16 product is exact in fp32, so each step equals the
// fp32 fma of the widened values -- the same sums as widening first, without
// the two conversions.
__device__ __forceinline__ void fma_sq_half2(uint32_t w, float &even, float &odd) {
    asm("{\n\t.reg .f16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "fma.rn.f32.f16 %0, lo, lo, %0;\n\t"
        "fma.rn.f32.f16 %1, hi, hi, %1;\n\t}"
        : "+f"(even), "+f"(odd)
        : "r"(w));
}

// Two E4M3 values -> their exact f16 pair, converted where it is used: the
// squared-sum pass converts each pair itself, so the compiler does not keep
// the converted pairs alive until the scaling pass (which converts again)
// and a thread can hold more vectors in flight.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_here(uint16_t two) {
    uint32_t h;
    asm volatile("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
    return h;
}

template <typename E>
struct HalfSquares {  // element types whose squares take fma_sq_half2
    static constexpr bool value = false;
};
template <>
struct HalfSquares<__half> {
    static constexpr bool value = true;
};
template <>
struct HalfSquares<__nv_fp8_e4m3> {
    static constexpr bool value = true;
};

template <typename E, int NV>
__device__ __forceinline__ float sumsq_pairs(const uint4 (&v)[NV]) {
    constexpr int K = Elem<E>::kPerVec / 2;
    if constexpr (HalfSquares<E>::value) {
        float even = 0.0f, odd = 0.0f;  // the two lanes of the f32x2 form below
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (sizeof(typename Elem<E>::Bits) == 2) {
                    fma_sq_half2(w[j], even, odd);
                } else {  // two E4M3 pairs per word, each widened exactly to f16x2
                    fma_sq_half2(e4m3x2_to_f16x2_here(static_cast<uint16_t>(w[j] & 0xFFFFu)), even, odd);
                    fma_sq_half2(e4m3x2_to_f16x2_here(static_cast<uint16_t>(w[j] >> 16)), even, odd);
                }
            }
        }
        return even + odd;
    } else {
        F2 acc = f2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            F2 x[K];
            Elem<E>::widen(v[i], x);
#pragma unroll
            for (int j = 0; j < K; ++j) acc = fma2(x[j], x[j], acc);
        }
        return f2_lo(acc) + f2_hi(acc);
    }
}

// Phase B on the way out, one vector: y = (x * gamma) * r, rounded once.
template <typename E>
__device__ __forceinline__ uint4 scale_vec(const uint4 &xv, const uint4 (&gv)[Elem<E>::kGVecs], F2 r2) {
    using GT = typename Elem<E>::G;
    constexpr int K = Elem<E>::kPerVec / 2;
    constexpr int KG = Elem<GT>::kPerVec / 2;
    F2 x[K], g[K];
    Elem<E>::widen(xv, x);
#pragma unroll
    for (int j = 0; j < Elem<E>::kGVecs; ++j) {
        F2 part[KG];
        Elem<GT>::widen(gv[j], part);
#pragma unroll
        for (int k = 0; k < KG; ++k) g[j * KG + k] = part[k];
    }
#pragma unroll
    for (int j = 0; j < K; ++j) x[j] = mul2(mul2(x[j], g[j]), r2);
    return Elem<E>::narrow(x);
}

// ----------------------------------------------------------------------------
// One-pass register kernel.
//
// A row (a token's Q or K row, or one head of it) is handled by a group of
// `group` threads -- 1, 2, 4, 8 or 16 lanes of a warp, or a multiple of 32
// that divides the CTA; a CTA of blockDim threads therefore handles
// rows_per_item = blockDim / group consecutive rows of one tensor per item.
// Items are the Q row-groups followed by the K row-groups (in a multi-shard
// launch: the row-groups of each Q shard, then of each K shard), and CTA c
// takes items c, c + grid, ...: every CTA gets a near-equal share of each
// tensor's rows whatever the grid.  Lane l of a group owns vectors l, l + group, ...
// (up to NV) of its row -- the same positions in every row -- so while
// consecutive items belong to one tensor a thread keeps that tensor's
// parameters and its gamma vectors in registers.  All loads of a row are
// issued before any is used.  A group of up to one warp reduces with shuffles
// only; wider groups add one CTA barrier per item.  Narrow rows (a K row
// beside a wide Q row, an attention head) thus share a CTA -- or a warp --
// instead of each paying for a whole one.
// TAIL: some row ends in a partial vector (otherwise the tail code is
// compiled out).
// Element types whose gamma vectors are re-read per row (through L1, where
// they stay: the same few KB for every row of a tensor) instead of being
// held in registers across rows.
template <typename E>
struct GammaPerRow {
    static constexpr bool value = false;
};
#ifndef QKN_E4M3_GAMMA_PER_ROW
#define QKN_E4M3_GAMMA_PER_ROW 1
#endif
template <>
struct GammaPerRow<__nv_fp8_e4m3> {
    static constexpr bool value = QKN_E4M3_GAMMA_PER_ROW != 0;
};

template <int NV>
struct RegisterBounds {
    static constexpr int kMaxThreads = NV <= 2 ? 1024 : (NV == 4 ? 512 : 256);
};

template <typename E, int NV, int MODE, bool TAIL, int SETS>
__global__ void __launch_bounds__(RegisterBounds<NV>::kMaxThreads)
    rows_register_kernel(const __grid_constant__ ParamsT<SETS> p) {
    constexpr int KG = Elem<E>::kGVecs;
    __shared__ float red[2][32];
    pdl_wait_and_release();
    int slot = 0;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t T = p.T;
    const int64_t n_items = p.n_items;
    const int64_t q_end = p.set[0].item_end;  // two sets (Q, K): the item where K starts

    int which = -1;
    int64_t set_begin = 0, set_end = 0;  // items of the current set: [set_begin, set_end)
    const char *in = nullptr;
    char *out = nullptr;
    float *sums = nullptr;
    const float *sums_all = nullptr;
    int64_t stride = 0, head_bytes = 0, rows = 0;
    int nfull = 0, tail = 0, gsize = 32, rpi = 1, grp = 0, gl = 0, gwarps = 1, heads = 1, nparts = 1;
    float inv_div = 0.0f;
    constexpr int NG = GammaPerRow<E>::value ? 1 : NV;  // gamma vectors held across rows
    uint4 g[NG][KG];
    const char *gamma = nullptr;

    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        bool next_set;  // uniform across the CTA: this item lies in another set than the last one
        if constexpr (SETS == 2) {
            const int w = item >= q_end ? 1 : 0;
            next_set = w != which;
            if (next_set) {
                which = w;
                set_begin = w ? q_end : 0;
            }
        } else {
            next_set = item >= set_end;
            if (next_set) {
                do {
                    ++which;
                    set_begin = set_end;
                    set_end = p.set[which].item_end;
                } while (item >= set_end);
            }
        }
        if (next_set) {
            const RowSet &d = p.set[which];
            in = d.in;
            out = d.out;
            sums = d.sumsq;
            sums_all = d.sumsq_all;
            nparts = d.P;
            stride = d.stride_bytes;
            head_bytes = d.head_bytes;
            heads = d.heads;
            rows = d.rows;
            nfull = d.nfull;
            tail = TAIL ? d.tail : 0;
            inv_div = d.inv_div;
            gsize = d.group;
            rpi = d.rows_per_item;
            grp = tid / gsize;
            gl = tid - grp * gsize;
            gwarps = gsize >> 5;
            if (MODE != kStats && !GammaPerRow<E>::value) {
#pragma unroll
                for (int i = 0; i < NV; ++i) ld_gamma_vec<E>(d.gamma, gl + i * gsize, nfull, tail, g[i]);
            }
            gamma = d.gamma;
        }
        const int64_t t = (item - set_begin) * rpi + grp;  // row index within the set (= token when heads == 1)
        const bool active = t < rows;
        const int64_t roff = active ? row_offset(t, heads, stride, head_bytes) : 0;
        const char *row = in + roff;
        uint4 v[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = gl + i * gsize;
            const int64_t off = static_cast<int64_t>(vi) * 16;
            if (active && vi < nfull)
                v[i] = ld_stream(row + off);
            else if (TAIL && active && vi == nfull && tail)
                v[i] = ld_tail<E>(row + off, tail);
            else
                v[i] = make_uint4(0u, 0u, 0u, 0u);
        }

        float r;
        if (MODE == kApply) {
            const float S = gsize < 32 ? combine_partials_lanes(sums_all, T, nparts, t, active, gl, gsize)
                                       : combine_partials_lanes(sums_all, T, nparts, t, active, lane, 32);
            r = active ? rms_factor(S, inv_div, p.eps) : 0.0f;
        } else {
            float S = sumsq_pairs<E, NV>(v);
            S = gsize < 32 ? segment_sum(S, gsize) : warp_sum(S);
            if (gwarps > 1) {  // uniform: the whole CTA takes this branch
                if (lane == 0) red[slot][warp] = S;
                __syncthreads();
                S = 0.0f;
                for (int k = 0; k < gwarps; ++k) S += red[slot][grp * gwarps + k];
                slot ^= 1;
            }
            if (MODE == kStats) {
                if (active && gl == 0) sums[t] = S;
                continue;
            }
            r = rms_factor(S, inv_div, p.eps);
        }
        if (!active) continue;
        const F2 r2 = f2(r, r);
        char *orow = out + roff;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = gl + i * gsize;
            const int64_t off = static_cast<int64_t>(vi) * 16;
            const bool full = vi < nfull;
            const bool part = TAIL && vi == nfull && tail;
            if (full || part) {
                uint4 y;
                if constexpr (GammaPerRow<E>::value) {
                    uint4 gv[KG];
                    ld_gamma_vec<E>(gamma, vi, nfull, tail, gv);
                    y = scale_vec<E>(v[i], gv, r2);
                } else {
                    y = scale_vec<E>(v[i], g[i < NG ? i : 0], r2);
                }
                if (full)
                    st_stream(orow + off, y);
                else
                    st_tail<E>(orow + off, y, tail);
            }
        }
    }
}

// ----------------------------------------------------------------------------
// Two-pass kernel for rows too wide for registers (VEC) or buffers that are
// not 16-byte aligned (!VEC, element-wise).  Pass 1 forms the squared sum;
// pass 2 re-reads x (largely from L2), scales and stores.  In place is safe:
// pass 2 reads each element before the same thread writes it, and pass 1 has
// finished for the whole row (block barrier) before pass 2 starts.  Items are
// whole rows, Q rows first, then K rows.
template <typename E, bool VEC, int MODE>
__global__ void __launch_bounds__(1024) rows_twopass_kernel(const __grid_constant__ Params p) {
    using EL = Elem<E>;
    using GT = typename EL::G;
    constexpr int K = EL::kPerVec / 2;
    __shared__ float red[2][32];
    pdl_wait_and_release();
    int slot = 0;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;

    const int64_t q_rows = p.set[0].rows;
    for (int64_t item = blockIdx.x; item < q_rows + p.set[1].rows; item += gridDim.x) {
        const int w = item >= q_rows ? 1 : 0;
        const RowSet &d = p.set[w];
        const int64_t t = w ? item - q_rows : item;  // row index (= token when heads == 1)
        const int64_t roff = row_offset(t, d.heads, d.stride_bytes, d.head_bytes);
        const char *row = d.in + roff;
        const int units = VEC ? d.nfull + (d.tail ? 1 : 0) : d.width;

        float r;
        if (MODE == kApply) {
            r = rms_factor(combine_partials_lanes(d.sumsq_all, p.T, d.P, t, true, tid & 31, 32), d.inv_div, p.eps);
        } else {
            float acc = 0.0f;
            for (int u = tid; u < units; u += nthr) {
                if (VEC) {
                    const uint4 v = (u < d.nfull) ? ld_stream(row + static_cast<int64_t>(u) * 16)
                                                  : ld_tail<E>(row + static_cast<int64_t>(u) * 16, d.tail);
                    F2 x[K];
                    EL::widen(v, x);
                    F2 a = f2(0.0f, 0.0f);
#pragma unroll
                    for (int j = 0; j < K; ++j) a = fma2(x[j], x[j], a);
                    acc += f2_lo(a) + f2_hi(a);
                } else {
                    const float f = EL::to_float(reinterpret_cast<const typename EL::Bits *>(row)[u]);
                    acc = fmaf(f, f, acc);
                }
            }
            const float S = block_sum(acc, red, slot);
            if (MODE == kStats) {
                if (tid == 0) d.sumsq[t] = S;
                continue;
            }
            r = rms_factor(S, d.inv_div, p.eps);
        }

        char *orow = d.out + roff;
        for (int u = tid; u < units; u += nthr) {
            if (VEC) {
                const bool full = u < d.nfull;
                const int64_t off = static_cast<int64_t>(u) * 16;
                const uint4 xv = full ? ld_stream(row + off) : ld_tail<E>(row + off, d.tail);
                uint4 gv[EL::kGVecs];
                ld_gamma_vec<E>(d.gamma, u, d.nfull, d.tail, gv);
                const uint4 y = scale_vec<E>(xv, gv, f2(r, r));
                if (full)
                    st_stream(orow + off, y);
                else
                    st_tail<E>(orow + off, y, d.tail);
            } else {
                const float f = EL::to_float(reinterpret_cast<const typename EL::Bits *>(row)[u]);
                const float g = Elem<GT>::to_float(reinterpret_cast<const typename Elem<GT>::Bits *>(d.gamma)[u]);
                reinterpret_cast<typename EL::Bits *>(orow)[u] = EL::from_float((f * g) * r);
            }
        }
    }
}

}  // namespace qkn
