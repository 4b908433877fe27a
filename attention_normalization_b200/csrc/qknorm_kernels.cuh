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
//
// The work is a read-once / write-once stream with a per-row reduction: no
// contraction, so no tensor cores.  What matters on B200 is bytes in flight
// per SM (16-byte coalesced vectors, several rows per SM outstanding), a short
// per-row critical path, and a grid bounded by residency.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {

enum Mode : int {
    kFused = 0,  // sum of squares -> factor -> scale and store
    kStats = 1,  // sum of squares -> write fp32 partial sum
    kApply = 2   // combine P partial sums -> factor -> scale and store
};

// One tensor's rows (Q or K, or a shard of one).
struct RowSet {
    const char *in;          // row t starts at in + t * stride_bytes
    char *out;               // kFused / kApply
    const char *gamma;       // kFused / kApply, [width]
    float *sumsq;            // kStats: [T]
    const float *sumsq_all;  // kApply: [P][T]
    int64_t stride_bytes;
    int32_t width;           // elements in this row (shard width for kStats / kApply)
    int32_t nfull;           // full 16-byte vectors in the row
    int32_t tail;            // elements after the last full vector
    float inv_div;           // 1 / (the FULL width), rounded to fp32 on the host
    int32_t group;           // register kernel: threads that share one row (a multiple of 32)
    int32_t rows_per_item;   // register kernel: blockDim / group rows handled per item
    int64_t items;           // register kernel: ceil(T / rows_per_item)
};

struct Params {
    RowSet set[2];           // 0 = Q, 1 = K
    int64_t T;
    float eps;
    int32_t P;               // kApply: number of shards
};

// ----------------------------------------------------------------------------
// Element packing: 16-byte vectors <-> fp32 lanes.
template <typename E>
struct Pack;

template <>
struct Pack<float> {
    static constexpr int N = 4;  // elements per 16-byte vector
    using Bits = uint32_t;
    __device__ __forceinline__ static void widen(const uint4 &v, float (&f)[N]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 narrow(const float (&f)[N]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
    __device__ __forceinline__ static float bits_to_float(Bits b) { return __uint_as_float(b); }
    __device__ __forceinline__ static Bits float_to_bits(float f) { return __float_as_uint(f); }
};

template <>
struct Pack<__nv_bfloat16> {
    static constexpr int N = 8;
    using Bits = uint16_t;
    // A bf16 value is the upper half of the fp32 with the same bits: widening is exact.
    __device__ __forceinline__ static void widen2(uint32_t u, float &lo, float &hi) {
        lo = __uint_as_float(u << 16);
        hi = __uint_as_float(u & 0xFFFF0000u);
    }
    __device__ __forceinline__ static uint32_t narrow2(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __device__ __forceinline__ static void widen(const uint4 &v, float (&f)[N]) {
        widen2(v.x, f[0], f[1]);
        widen2(v.y, f[2], f[3]);
        widen2(v.z, f[4], f[5]);
        widen2(v.w, f[6], f[7]);
    }
    __device__ __forceinline__ static uint4 narrow(const float (&f)[N]) {
        return make_uint4(narrow2(f[0], f[1]), narrow2(f[2], f[3]), narrow2(f[4], f[5]),
                          narrow2(f[6], f[7]));
    }
    __device__ __forceinline__ static float bits_to_float(Bits b) {
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    __device__ __forceinline__ static Bits float_to_bits(float f) {
        return __bfloat16_as_ushort(__float2bfloat16_rn(f));
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

// The last, partial vector of a row: `n` (< N) elements, the rest zero.
template <typename E>
__device__ __forceinline__ uint4 ld_tail(const char *p, int n) {
    using P = Pack<E>;
    typename P::Bits b[P::N];
    const typename P::Bits *src = reinterpret_cast<const typename P::Bits *>(p);
#pragma unroll
    for (int e = 0; e < P::N; ++e) b[e] = (e < n) ? src[e] : typename P::Bits(0);
    uint4 v;
    static_assert(sizeof(b) == sizeof(uint4), "vector size");
    memcpy(&v, b, sizeof(v));
    return v;
}
template <typename E>
__device__ __forceinline__ void st_tail(char *p, const uint4 &v, int n) {
    using P = Pack<E>;
    typename P::Bits b[P::N];
    memcpy(b, &v, sizeof(v));
    typename P::Bits *dst = reinterpret_cast<typename P::Bits *>(p);
#pragma unroll
    for (int e = 0; e < P::N; ++e)
        if (e < n) dst[e] = b[e];
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

// Phase A aggregation: the P partial sums of token t, added in order p = 0..P-1.
__device__ __forceinline__ float combine_partials(const float *all, int64_t T, int P, int64_t t) {
    float s = 0.0f;
    for (int p = 0; p < P; ++p) s += __ldg(all + static_cast<int64_t>(p) * T + t);
    return s;
}

// r = 1 / sqrt(S / H + eps), the mean formed as S * fl(1 / H).
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

__device__ __forceinline__ float rms_factor(float sumsq, float inv_div, float eps) {
    return rsqrtf(sumsq * inv_div + eps);
}

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

// A 16-byte vector as fp32 pairs: bf16 holds 4 pairs (one per 32-bit word),
// fp32 holds 2.
template <typename E>
struct Pairs;
template <>
struct Pairs<__nv_bfloat16> {
    static constexpr int K = 4;
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[K]) {
        // the bf16 in the low half of a word is the fp32 with those bits in the high half
        p[0] = f2_bits(v.x << 16, v.x & 0xFFFF0000u);
        p[1] = f2_bits(v.y << 16, v.y & 0xFFFF0000u);
        p[2] = f2_bits(v.z << 16, v.z & 0xFFFF0000u);
        p[3] = f2_bits(v.w << 16, v.w & 0xFFFF0000u);
    }
    __device__ __forceinline__ static uint32_t narrow1(F2 a) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f2_lo(a), f2_hi(a));  // round to nearest even
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[K]) {
        return make_uint4(narrow1(p[0]), narrow1(p[1]), narrow1(p[2]), narrow1(p[3]));
    }
};
template <>
struct Pairs<float> {
    static constexpr int K = 2;
    __device__ __forceinline__ static void widen(const uint4 &v, F2 (&p)[K]) {
        p[0] = f2_bits(v.x, v.y);
        p[1] = f2_bits(v.z, v.w);
    }
    __device__ __forceinline__ static uint4 narrow(const F2 (&p)[K]) {
        return make_uint4(static_cast<uint32_t>(p[0].v), static_cast<uint32_t>(p[0].v >> 32),
                          static_cast<uint32_t>(p[1].v), static_cast<uint32_t>(p[1].v >> 32));
    }
};

// Squared sum of a thread's vectors (two fp32 lanes accumulate the even and
// odd elements; they are added at the end).
template <typename E, int NV>
__device__ __forceinline__ float sumsq_pairs(const uint4 (&v)[NV]) {
    using PP = Pairs<E>;
    F2 acc = f2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        F2 x[PP::K];
        PP::widen(v[i], x);
#pragma unroll
        for (int j = 0; j < PP::K; ++j) acc = fma2(x[j], x[j], acc);
    }
    return f2_lo(acc) + f2_hi(acc);
}

// Phase B on the way out, one vector: y = (x * gamma) * r, rounded once.
template <typename E>
__device__ __forceinline__ uint4 scale_vec(const uint4 &xv, const uint4 &gv, F2 r2) {
    using PP = Pairs<E>;
    F2 x[PP::K], g[PP::K];
    PP::widen(xv, x);
    PP::widen(gv, g);
#pragma unroll
    for (int j = 0; j < PP::K; ++j) x[j] = mul2(mul2(x[j], g[j]), r2);
    return PP::narrow(x);
}

// ----------------------------------------------------------------------------
// One-pass register kernel.
//
// A row is handled by a group of `group` threads (a multiple of 32 that
// divides the CTA); a CTA of blockDim threads therefore handles
// rows_per_item = blockDim / group consecutive rows of one tensor per item.
// Items are the Q row-groups followed by the K row-groups, and CTA c takes
// items c, c + grid, ...: every CTA gets a near-equal share of each tensor's
// rows whatever the grid.  Lane l of a group owns vectors l, l + group, ...
// (up to NV) of its row -- the same positions in every row -- so while
// consecutive items belong to one tensor a thread keeps that tensor's
// parameters and its gamma vectors in registers.  All loads of a row are
// issued before any is used.  A one-warp group reduces with shuffles only;
// wider groups add one CTA barrier per item.  Narrow rows (e.g. K beside a
// wide Q) thus share a CTA instead of each paying for a whole one.
// TAIL: some row ends in a partial vector (otherwise the tail code is
// compiled out).
template <int NV>
struct RegisterBounds {
    static constexpr int kMaxThreads = NV <= 2 ? 1024 : (NV == 4 ? 512 : 256);
};

template <typename E, int NV, int MODE, bool TAIL>
__global__ void __launch_bounds__(RegisterBounds<NV>::kMaxThreads)
    rows_register_kernel(const __grid_constant__ Params p) {
    __shared__ float red[2][32];
    pdl_wait_and_release();
    int slot = 0;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t T = p.T;
    const int64_t q_items = p.set[0].items;
    const int64_t n_items = q_items + p.set[1].items;

    int which = -1;
    const char *in = nullptr;
    char *out = nullptr;
    float *sums = nullptr;
    const float *sums_all = nullptr;
    int64_t stride = 0;
    int nfull = 0, tail = 0, gsize = 32, rpi = 1, grp = 0, gl = 0, gwarps = 1;
    float inv_div = 0.0f;
    uint4 g[NV];

    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int w = item >= q_items ? 1 : 0;
        const int64_t j = w ? item - q_items : item;
        if (w != which) {  // uniform across the CTA
            which = w;
            const RowSet &d = p.set[w];
            in = d.in;
            out = d.out;
            sums = d.sumsq;
            sums_all = d.sumsq_all;
            stride = d.stride_bytes;
            nfull = d.nfull;
            tail = TAIL ? d.tail : 0;
            inv_div = d.inv_div;
            gsize = d.group;
            rpi = d.rows_per_item;
            grp = tid / gsize;
            gl = tid - grp * gsize;
            gwarps = gsize >> 5;
            if (MODE != kStats) {
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int vi = gl + i * gsize;
                    const int64_t off = static_cast<int64_t>(vi) * 16;
                    if (vi < nfull)
                        g[i] = ld_gamma(d.gamma + off);
                    else if (TAIL && vi == nfull && tail)
                        g[i] = ld_tail<E>(d.gamma + off, tail);
                    else
                        g[i] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        const int64_t t = j * rpi + grp;
        const bool active = t < T;
        const char *row = in + t * stride;
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
            r = active ? rms_factor(combine_partials(sums_all, T, p.P, t), inv_div, p.eps) : 0.0f;
        } else {
            float S = warp_sum(sumsq_pairs<E, NV>(v));
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
        char *orow = out + t * stride;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = gl + i * gsize;
            const int64_t off = static_cast<int64_t>(vi) * 16;
            if (vi < nfull)
                st_stream(orow + off, scale_vec<E>(v[i], g[i], r2));
            else if (TAIL && vi == nfull && tail)
                st_tail<E>(orow + off, scale_vec<E>(v[i], g[i], r2), tail);
        }
    }
}

// ----------------------------------------------------------------------------
// Two-pass kernel for rows too wide for registers (VEC) or buffers that are
// not 16-byte aligned (!VEC, element-wise).  Pass 1 forms the squared sum;
// pass 2 re-reads x (largely from L2), scales and stores.  In place is safe:
// pass 2 reads each element before the same thread writes it, and pass 1 has
// finished for the whole row (block barrier) before pass 2 starts.
template <typename E, bool VEC, int MODE>
__global__ void __launch_bounds__(1024) rows_twopass_kernel(const __grid_constant__ Params p) {
    using Pk = Pack<E>;
    __shared__ float red[2][32];
    pdl_wait_and_release();
    int slot = 0;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;

    for (int64_t item = blockIdx.x; item < 2 * p.T; item += gridDim.x) {
        const int w = item >= p.T ? 1 : 0;  // Q rows first, then K rows
        const RowSet &d = p.set[w];
        const int64_t t = w ? item - p.T : item;
        const char *row = d.in + t * d.stride_bytes;
        const int units = VEC ? d.nfull + (d.tail ? 1 : 0) : d.width;

        float r;
        if (MODE == kApply) {
            r = rms_factor(combine_partials(d.sumsq_all, p.T, p.P, t), d.inv_div, p.eps);
        } else {
            float acc = 0.0f;
            for (int u = tid; u < units; u += nthr) {
                if (VEC) {
                    const uint4 v = (u < d.nfull) ? ld_stream(row + static_cast<int64_t>(u) * 16)
                                                  : ld_tail<E>(row + static_cast<int64_t>(u) * 16, d.tail);
                    float f[Pk::N];
                    Pk::widen(v, f);
#pragma unroll
                    for (int e = 0; e < Pk::N; ++e) acc = fmaf(f[e], f[e], acc);
                } else {
                    const float f = Pk::bits_to_float(
                        reinterpret_cast<const typename Pk::Bits *>(row)[u]);
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

        char *orow = d.out + t * d.stride_bytes;
        for (int u = tid; u < units; u += nthr) {
            if (VEC) {
                const bool full = u < d.nfull;
                const int64_t off = static_cast<int64_t>(u) * 16;
                const uint4 xv = full ? ld_stream(row + off) : ld_tail<E>(row + off, d.tail);
                const uint4 gv = full ? ld_gamma(d.gamma + off) : ld_tail<E>(d.gamma + off, d.tail);
                float f[Pk::N], g[Pk::N];
                Pk::widen(xv, f);
                Pk::widen(gv, g);
#pragma unroll
                for (int e = 0; e < Pk::N; ++e) f[e] = (f[e] * g[e]) * r;
                const uint4 y = Pk::narrow(f);
                if (full)
                    st_stream(orow + off, y);
                else
                    st_tail<E>(orow + off, y, d.tail);
            } else {
                const float f = Pk::bits_to_float(reinterpret_cast<const typename Pk::Bits *>(row)[u]);
                const float g =
                    Pk::bits_to_float(reinterpret_cast<const typename Pk::Bits *>(d.gamma)[u]);
                reinterpret_cast<typename Pk::Bits *>(orow)[u] = Pk::float_to_bits((f * g) * r);
            }
        }
    }
}

}  // namespace qkn
