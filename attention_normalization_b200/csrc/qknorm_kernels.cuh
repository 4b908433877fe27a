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
//     loop over tokens (here: over Q and K row items).
//
// The work is a read-once / write-once stream with a per-row reduction: no
// contraction, so no tensor cores.  What matters on B200 is bytes in flight
// per SM (16-byte coalesced vector loads, several rows per SM resident), a
// short per-row critical path, and a grid bounded by residency.
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
    float div;               // divisor of the mean: the FULL width, as float
};

struct Params {
    RowSet set[2];  // 0 = Q, 1 = K
    int64_t T;
    int64_t rows;   // 2 * T row items
    float eps;
    int32_t P;      // kApply: number of shards
};

// ----------------------------------------------------------------------------
// Element packing: 16-byte vectors <-> fp32 lanes.
template <typename E>
struct Pack;

template <>
struct Pack<float> {
    static constexpr int N = 4;  // elements per 16-byte vector
    static constexpr int kBytes = 4;
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
    static constexpr int kBytes = 2;
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
// lets one __syncthreads per row suffice: a thread can only overwrite slot s
// after every thread has passed the barrier of the row in between, i.e. after
// all reads of slot s are done.
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

__device__ __forceinline__ float rms_factor(float sumsq, float div, float eps) {
    return rsqrtf(sumsq / div + eps);
}

// ----------------------------------------------------------------------------
// One-pass register kernel.  Each CTA holds one row at a time in registers:
// thread i owns vectors i, i + blockDim, ..., up to NV of them.  All loads of
// a row are issued before any is used.
template <int NV>
struct RegisterBounds {
    static constexpr int kMaxThreads = NV <= 2 ? 1024 : (NV == 4 ? 512 : 256);
};

template <typename E, int NV, int MODE>
__global__ void __launch_bounds__(RegisterBounds<NV>::kMaxThreads)
    rows_register_kernel(const __grid_constant__ Params p) {
    using Pk = Pack<E>;
    __shared__ float red[2][32];
    int slot = 0;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;

    for (int64_t item = blockIdx.x; item < p.rows; item += gridDim.x) {
        const RowSet &d = p.set[item & 1];
        const int64_t t = item >> 1;
        const char *row = d.in + t * d.stride_bytes;

        uint4 v[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = tid + i * nthr;
            if (vi < d.nfull)
                v[i] = ld_stream(row + static_cast<int64_t>(vi) * 16);
            else if (vi == d.nfull && d.tail)
                v[i] = ld_tail<E>(row + static_cast<int64_t>(vi) * 16, d.tail);
            else
                v[i] = make_uint4(0u, 0u, 0u, 0u);
        }

        float r;
        if (MODE == kApply) {
            r = rms_factor(combine_partials(d.sumsq_all, p.T, p.P, t), d.div, p.eps);
        } else {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                float f[Pk::N];
                Pk::widen(v[i], f);
#pragma unroll
                for (int e = 0; e < Pk::N; ++e) acc = fmaf(f[e], f[e], acc);
            }
            const float S = block_sum(acc, red, slot);
            if (MODE == kStats) {
                if (tid == 0) d.sumsq[t] = S;
                continue;
            }
            r = rms_factor(S, d.div, p.eps);
        }

        char *orow = d.out + t * d.stride_bytes;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = tid + i * nthr;
            const bool full = vi < d.nfull;
            const bool part = (vi == d.nfull) && d.tail;
            if (full || part) {
                const uint4 gv = full ? ld_gamma(d.gamma + static_cast<int64_t>(vi) * 16)
                                      : ld_tail<E>(d.gamma + static_cast<int64_t>(vi) * 16, d.tail);
                float f[Pk::N], g[Pk::N];
                Pk::widen(v[i], f);
                Pk::widen(gv, g);
#pragma unroll
                for (int e = 0; e < Pk::N; ++e) f[e] = (f[e] * g[e]) * r;
                const uint4 y = Pk::narrow(f);
                if (full)
                    st_stream(orow + static_cast<int64_t>(vi) * 16, y);
                else
                    st_tail<E>(orow + static_cast<int64_t>(vi) * 16, y, d.tail);
            }
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
    int slot = 0;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;

    for (int64_t item = blockIdx.x; item < p.rows; item += gridDim.x) {
        const RowSet &d = p.set[item & 1];
        const int64_t t = item >> 1;
        const char *row = d.in + t * d.stride_bytes;
        const int units = VEC ? d.nfull + (d.tail ? 1 : 0) : d.width;

        float r;
        if (MODE == kApply) {
            r = rms_factor(combine_partials(d.sumsq_all, p.T, p.P, t), d.div, p.eps);
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
            r = rms_factor(S, d.div, p.eps);
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
