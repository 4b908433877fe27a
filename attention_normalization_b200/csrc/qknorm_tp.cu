// Tensor-parallel layerwise QK-Norm with the scalar partial sums exchanged
// through memory (structure and protocol in qknorm_tp.cuh).

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "qknorm_kernels.cuh"
#include "qknorm_tp.cuh"

namespace qkn {
namespace tp {
namespace {

// Set to 4 by a wait that ran out or gave up (every wait that returns without
// its partial sums sets it); read and cleared by the host.
__device__ int g_tp_timeout = 0;

// Memory scope of the exchange: system when some ranks are on other GPUs
// (peer memory), GPU when every rank runs in this launch.

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned long long pack(uint32_t epoch, float v) {
    return (static_cast<unsigned long long>(epoch) << 32) | __float_as_uint(v);
}

// The abort word of a receive buffer: the 64-bit word after its [R][T][2]
// exchange words.  A wait that runs out stores the call's epoch there, in the
// buffer of every rank of its launch, and the other waits of that call give
// up when they see it.  It belongs to the buffer set and the epoch together,
// so a later call -- a later epoch on these buffers, or any epoch on another
// (zeroed) set -- never mistakes an old abort for its own.
__device__ __forceinline__ unsigned long long *abort_word(const TpParams &p, int rank) {
    return p.recv[rank] + static_cast<int64_t>(p.R) * p.T * 2;
}

template <bool SYS>
__device__ __forceinline__ bool aborted(const unsigned long long *word, uint32_t epoch) {
    unsigned long long v;
    if constexpr (SYS)
        asm volatile("ld.relaxed.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(word) : "memory");
    else
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(word) : "memory");
    return v == epoch;
}

// Marks the call aborted in the abort word of every rank this launch runs.
template <bool SYS>
__device__ __forceinline__ void mark_aborted(const TpParams &p, uint32_t epoch) {
    for (int j = 0; j < p.n_local; ++j) {
        unsigned long long *w = abort_word(p, p.first_rank + j);
        const unsigned long long v = epoch;
        if constexpr (SYS)
            asm volatile("st.relaxed.sys.global.u64 [%0], %1;" ::"l"(w), "l"(v) : "memory");
        else
            asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(w), "l"(v) : "memory");
    }
}

// Publishes this rank's partial sums for one token (the Q word, then the K
// word, one 16-byte store).  Each word carries the call's epoch beside its
// value, so a reader that sees the epoch in a word has that word's value:
// nothing else is communicated, so no ordering between the words or with
// other memory is needed and relaxed stores suffice.
template <bool SYS>
__device__ __forceinline__ void publish_pair(unsigned long long *dst, uint32_t epoch, float sq, float sk) {
    const unsigned long long wq = pack(epoch, sq), wk = pack(epoch, sk);
    if constexpr (SYS)
        asm volatile("st.relaxed.sys.global.v2.u64 [%0], {%1, %2};" ::"l"(dst), "l"(wq), "l"(wk) : "memory");
    else
        asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(dst), "l"(wq), "l"(wk) : "memory");
}

template <bool SYS>
__device__ __forceinline__ void load_pair(const unsigned long long *src, unsigned long long &wq,
                                          unsigned long long &wk) {
    if constexpr (SYS)
        asm volatile("ld.relaxed.sys.global.v2.u64 {%0, %1}, [%2];" : "=l"(wq), "=l"(wk) : "l"(src) : "memory");
    else
        asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(wq), "=l"(wk) : "l"(src) : "memory");
}

// Waits (bounded) until both words at `src` carry the call's epoch; their
// values, or false after a timeout or an abort of this call (`rank` is the
// waiting rank, whose buffer holds the abort word it watches).  Every false
// return records code 4.
template <bool SYS>
__device__ __forceinline__ bool wait_pair(const TpParams &p, int rank, const unsigned long long *src, float &vq,
                                          float &vk) {
    const uint32_t epoch = p.epoch;
    unsigned long long wq, wk;
    load_pair<SYS>(src, wq, wk);
    if (static_cast<uint32_t>(wq >> 32) != epoch || static_cast<uint32_t>(wk >> 32) != epoch) {
        const uint64_t t0 = now_ns();
        const unsigned long long *abort = abort_word(p, rank);
        for (uint32_t it = 1;; ++it) {
            __nanosleep(32);
            load_pair<SYS>(src, wq, wk);
            if (static_cast<uint32_t>(wq >> 32) == epoch && static_cast<uint32_t>(wk >> 32) == epoch) break;
            // every waiting lane of a rank would read the same abort word:
            // look at it (and the clock) every 64 polls only
            if ((it & 63u) == 0) {
                const bool gave_up = aborted<SYS>(abort, epoch);
                if (gave_up || now_ns() - t0 > p.timeout_ns) {
                    atomicExch(&g_tp_timeout, 4);
                    if (!gave_up) mark_aborted<SYS>(p, epoch);
                    return false;
                }
            }
        }
    }
    vq = __uint_as_float(static_cast<uint32_t>(wq));
    vk = __uint_as_float(static_cast<uint32_t>(wk));
    return true;
}

}  // namespace

// One warp per token, kTpWarps warps per block, no block barrier.  Warp w of
// block c of a rank takes tokens (c * kTpWarps + w), + G * kTpWarps, ...;
// lane i exchanges with rank i, every lane gets the sums by shuffles, and
// the warp scales its row as (x * gamma) * r.  The exchange is a round trip
// through memory, so throughput comes from the number of tokens in flight: a
// warp passes its row through registers in batches of at most kTpBatch
// 16-byte vectors per lane (gamma re-read from L1 when the row is scaled)
// and publishes ahead, and the register cap below fits as many warps on an
// SM as one batch's registers allow.  Shard rows of up to 8 vectors per lane
// (NVQ for Q, NVK <= NVQ for K) run fully unrolled; wider rows take the
// kTpWide instantiation, whose batch loop runs over the row at run time.
constexpr int kTpWarps = 4;

#ifndef QKN_TP_AHEAD
#define QKN_TP_AHEAD 2
#endif
constexpr int kTpAhead = QKN_TP_AHEAD;  // tokens a warp publishes ahead of the one it finishes

#ifndef QKN_TP_BATCH
#define QKN_TP_BATCH 4
#endif
// 16-byte vectors per lane a warp loads at once: a row passes through the
// warp in batches, so registers depend on the batch, not on the row width.
constexpr int kTpBatch = QKN_TP_BATCH;

#ifndef QKN_TP_REGS_PER_VEC
#define QKN_TP_REGS_PER_VEC 4
#endif
constexpr int kTpWide = 0;  // NVQ = NVK = kTpWide: any width, batches of kTpBatch

template <int NVQ, int NVK>
constexpr int tp_warp_min_blocks() {
    // registers per 16-byte vector held (a batch of Q or K vectors, NVK <=
    // NVQ, and their gamma vectors), plus ~40 for the rest
    constexpr int held = 2 * (NVQ == kTpWide || NVQ > kTpBatch ? kTpBatch : NVQ);
    constexpr int regs = QKN_TP_REGS_PER_VEC * held + 40;
    return 65536 / (32 * kTpWarps * regs) < 16 ? 65536 / (32 * kTpWarps * regs) : 16;
}

// KEEP: the row will be read again soon (kept in L2 at normal priority);
// else its last read (streaming).
template <bool KEEP>
__device__ __forceinline__ uint4 tp_ld(const char *p) {
    if constexpr (KEEP)
        return __ldcg(reinterpret_cast<const uint4 *>(p));
    else
        return ld_stream(p);
}

template <int NV, bool KEEP, int B>
__device__ __forceinline__ void tp_load_batch(const char *row, int nvecs, int lane, int b, uint4 (&x)[B]) {
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const int vi = lane + 32 * (b + i);
        x[i] = vi < nvecs ? tp_ld<KEEP>(row + static_cast<int64_t>(vi) * 16) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Phase A, local step and publication: the shard's squared sums, Q and K
// batches loaded side by side, written to every rank's receive buffer (lane
// i to rank i).
template <typename E, int NVQ, int NVK, bool SYS>
__device__ __forceinline__ void tp_publish(const TpParams &p, const RankPtrs &rp, int rank, int64_t t, int lane) {
    constexpr int BQ = NVQ == kTpWide || NVQ > kTpBatch ? kTpBatch : NVQ;
    constexpr int BK = NVK == kTpWide || NVK > kTpBatch ? kTpBatch : NVK;
    const char *qrow = rp.q_in + t * p.q_stride_bytes;
    const char *krow = rp.k_in + t * p.k_stride_bytes;
    // vectors per lane of the wider row (Q; either for the wide form)
    const int nq = NVQ != kTpWide ? NVQ : ((p.q_vecs > p.k_vecs ? p.q_vecs : p.k_vecs) + 31) >> 5;
    float sq = 0.0f, sk = 0.0f;
#pragma unroll
    for (int b = 0; b < nq; b += BQ) {  // NVK <= NVQ
        uint4 xq[BQ], xk[BK];
        tp_load_batch<NVQ, true, BQ>(qrow, p.q_vecs, lane, b, xq);
        if (NVK == kTpWide || b < NVK) tp_load_batch<NVK, true, BK>(krow, p.k_vecs, lane, b, xk);
        sq += sumsq_pairs<E, BQ>(xq);
        if (NVK == kTpWide || b < NVK) sk += sumsq_pairs<E, BK>(xk);
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    if (lane < p.R) publish_pair<SYS>(p.recv[lane] + (static_cast<int64_t>(rank) * p.T + t) * 2, p.epoch, sq, sk);
}

// Phase B for one shard row, from its first batch (already loaded) on:
// (x * gamma) * r, batch by batch.
template <typename E, int NV, int B>
__device__ __forceinline__ void tp_scale_row(const char *in, char *out, const char *gamma, int nvecs, int lane,
                                             F2 r, uint4 (&x)[B]) {
    constexpr int KG = Elem<E>::kGVecs;
    const int nv = NV != kTpWide ? NV : (nvecs + 31) >> 5;
#pragma unroll
    for (int b = 0; b < nv; b += B) {
        if (b > 0) tp_load_batch<NV, false, B>(in, nvecs, lane, b, x);
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int vi = lane + 32 * (b + i);
            if (vi < nvecs) {
                uint4 g[KG];
                ld_gamma_vec<E>(gamma, vi, nvecs, 0, g);
                st_stream(out + static_cast<int64_t>(vi) * 16, scale_vec<E>(x[i], g, r));
            }
        }
    }
}

// Waits for the other ranks' partials of token t, adds them in rank order
// and stores (x * gamma) * r, re-reading the rows (the first batches of Q and
// K while the exchange completes); a wait that gave up leaves the token unwritten
// (the timeout is reported).
template <typename E, int NVQ, int NVK, bool SYS>
__device__ __forceinline__ void tp_finish(const TpParams &p, const RankPtrs &rp, int rank, int64_t t, int lane) {
    constexpr int BQ = NVQ == kTpWide || NVQ > kTpBatch ? kTpBatch : NVQ;
    constexpr int BK = NVK == kTpWide || NVK > kTpBatch ? kTpBatch : NVK;
    const char *qrow = rp.q_in + t * p.q_stride_bytes;
    const char *krow = rp.k_in + t * p.k_stride_bytes;
    uint4 xq[BQ], xk[BK];
    tp_load_batch<NVQ, false, BQ>(qrow, p.q_vecs, lane, 0, xq);
    tp_load_batch<NVK, false, BK>(krow, p.k_vecs, lane, 0, xk);
    float vq = 0.0f, vk = 0.0f;
    bool ok = true;
    if (lane < p.R)
        ok = wait_pair<SYS>(p, rank, p.recv[rank] + (static_cast<int64_t>(lane) * p.T + t) * 2, vq, vk);
    if (!__all_sync(0xFFFFFFFFu, ok)) return;  // a wait gave up: token left unwritten (reported)
    float Aq = 0.0f, Ak = 0.0f;  // Phase A aggregation, in rank order
    for (int i = 0; i < p.R; ++i) {
        Aq += __shfl_sync(0xFFFFFFFFu, vq, i);
        Ak += __shfl_sync(0xFFFFFFFFu, vk, i);
    }
    const float rq = rms_factor(Aq, p.inv_hq, p.eps), rk = rms_factor(Ak, p.inv_hk, p.eps);
    tp_scale_row<E, NVQ, BQ>(qrow, rp.q_out + t * p.q_stride_bytes, rp.gamma_q, p.q_vecs, lane, f2(rq, rq), xq);
    tp_scale_row<E, NVK, BK>(krow, rp.k_out + t * p.k_stride_bytes, rp.gamma_k, p.k_vecs, lane, f2(rk, rk), xk);
}

// Warp w of block c takes tokens s, s + step, s + 2 step, ... (s = c * 4 + w,
// step = G * 4) and publishes kTpAhead tokens ahead of the one it finishes:
// iteration k reads token k (kept in L2) and publishes its partial sums, then
// re-reads token k - kTpAhead (an L2 hit, read kTpAhead tokens earlier),
// waits for that token's exchange (by now mostly complete) and stores it.
// No row is held across a wait on the exchange beyond one batch.  Every
// rank's warp (c, w) has the same sequence and publishes a token before it
// waits on it, so no wait depends on a warp that waits on it.
template <typename E, int NVQ, int NVK, bool SYS>
__global__ void __launch_bounds__(32 * kTpWarps, tp_warp_min_blocks<NVQ, NVK>())
    tp_warp_kernel(const __grid_constant__ TpParams p) {
    pdl_wait_and_release();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int local = blockIdx.x / p.blocks_per_rank;
    const int c = blockIdx.x - local * p.blocks_per_rank;
    const int rank = p.first_rank + local;
    const RankPtrs rp = p.local[local];
    const int64_t step = static_cast<int64_t>(p.blocks_per_rank) * kTpWarps;
    const int64_t first = static_cast<int64_t>(c) * kTpWarps + warp;
    const int64_t n = first < p.T ? (p.T - 1 - first) / step + 1 : 0;  // tokens of this warp
    for (int64_t k = 0; k < n + kTpAhead; ++k) {
        if (k < n) tp_publish<E, NVQ, NVK, SYS>(p, rp, rank, first + k * step, lane);
        if (k >= kTpAhead) tp_finish<E, NVQ, NVK, SYS>(p, rp, rank, first + (k - kTpAhead) * step, lane);
    }
}

namespace {

// nv < 0: the warp kernel with NVQ and NVK vectors per lane, nv = -(8 NVQ +
// NVK); nv == 0: the warp kernel for rows of any width.
template <typename E, bool SYS>
const void *tp_kernel(int nv) {
    switch (nv) {
        case 0: return (const void *)tp_warp_kernel<E, kTpWide, kTpWide, SYS>;
        // nv = -(8 * NVQ + NVK), NVK <= NVQ (wider K rows take NVQ = NVK)
        case -(8 * 1 + 1): return (const void *)tp_warp_kernel<E, 1, 1, SYS>;
        case -(8 * 2 + 1): return (const void *)tp_warp_kernel<E, 2, 1, SYS>;
        case -(8 * 2 + 2): return (const void *)tp_warp_kernel<E, 2, 2, SYS>;
        case -(8 * 4 + 1): return (const void *)tp_warp_kernel<E, 4, 1, SYS>;
        case -(8 * 4 + 2): return (const void *)tp_warp_kernel<E, 4, 2, SYS>;
        case -(8 * 4 + 4): return (const void *)tp_warp_kernel<E, 4, 4, SYS>;
        case -(8 * 8 + 1): return (const void *)tp_warp_kernel<E, 8, 1, SYS>;
        case -(8 * 8 + 2): return (const void *)tp_warp_kernel<E, 8, 2, SYS>;
        case -(8 * 8 + 4): return (const void *)tp_warp_kernel<E, 8, 4, SYS>;
        case -(8 * 8 + 8): return (const void *)tp_warp_kernel<E, 8, 8, SYS>;
        default: return nullptr;
    }
}

template <bool SYS>
const void *tp_kernel(int dtype, int nv) {
    switch (dtype) {
        case 0: return tp_kernel<float, SYS>(nv);
        case 1: return tp_kernel<__nv_bfloat16, SYS>(nv);
        case 2: return tp_kernel<__half, SYS>(nv);
        case 3: return tp_kernel<__nv_fp8_e4m3, SYS>(nv);
        default: return nullptr;
    }
}

// GPU scope when every rank of the group runs in the launch, system scope
// when some rank runs elsewhere (peer memory).
const void *tp_kernel(int dtype, int nv, bool gpu_scope) {
    return gpu_scope ? tp_kernel<false>(dtype, nv) : tp_kernel<true>(dtype, nv);
}

}  // namespace

cudaError_t tp_blocks_per_sm(int dtype, int nv, int threads, bool gpu_scope, int *out) {
    const void *fn = tp_kernel(dtype, nv, gpu_scope);
    if (!fn) return cudaErrorInvalidValue;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, fn, threads, 0);
}

cudaError_t launch_tp(const TpParams &p, int dtype, int nv, int threads, bool gpu_scope, cudaStream_t stream,
                      const char **what) {
    if (gpu_scope && p.n_local != p.R) {
        *what = "GPU-scope exchange with ranks outside the launch";
        return cudaErrorInvalidValue;
    }
    const void *fn = tp_kernel(dtype, nv, gpu_scope);
    if (!fn) {
        *what = "kernel selection";
        return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.blocks_per_rank * p.n_local));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (p.n_local > 1) {  // blocks of different ranks wait on one another: all must be resident
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    void *args[] = {const_cast<TpParams *>(&p)};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) *what = "cudaLaunchKernelExC";
    return e;
}

cudaError_t tp_read_and_clear_timeout(int *code) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_tp_timeout, sizeof(int))) != cudaSuccess) return e;
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_tp_timeout, &zero, sizeof(int))) != cudaSuccess) return e;
    *code = v;
    return cudaSuccess;
}

}  // namespace tp
}  // namespace qkn
