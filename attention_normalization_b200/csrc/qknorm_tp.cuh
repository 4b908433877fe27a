// Tensor-parallel layerwise QK-Norm with the partial squared sums exchanged
// between ranks through memory (the paper's Phase A / Phase B kernel).
//
// Method: "SwiftQK: Fast and Communication-Efficient Tensor Parallelism for
// Query-Key Normalization" (arXiv 2608.09160).
//   Phase A: each rank holds a hidden-dimension shard of every token's Q and
//     K rows; it computes the shard's squared sums and the ranks add their
//     partial sums (fp32) to get the global sums -- a scalar per token and
//     tensor crosses between ranks instead of the activations.
//   Phase B: the shard times gamma is scaled by the global factor and only
//     the final values are stored.  The pages overlap the exchange with the
//     gamma multiply (warp 0 exchanges while the other warps multiply); here
//     one warp carries a token (four per block, no block barrier) and the
//     overlap is deeper: a warp publishes two tokens ahead of the one it
//     finishes and re-reads that one's rows from L2, so its exchange is
//     mostly complete when the warp waits on it, and no row is held across a
//     wait (rows pass through registers in batches, so any shard width fits).
//   Deadlock-safe persistent execution: the grid is bounded by the resident
//     blocks and each block loops over tokens.
//
// One kernel serves two deployments:
//   * one rank per GPU: each GPU launches its own rank; receive buffers of the
//     other ranks are reached through peer mappings (P2P stores and loads at
//     system scope);
//   * several ranks in one launch on one GPU (the test form here): the ranks'
//     blocks wait on one another, so the launch is cooperative (all blocks
//     resident at once).
// In both, block c of every rank processes tokens c, c + G, c + 2G, ... (G
// blocks per rank, equal on every rank) and publishes before it waits, so the
// blocks a wait depends on are never themselves waiting on it.
//
// Exchange format: rank i's receive buffer holds [R][T][2] 64-bit words; word
// (r, t, w) = (epoch << 32) | bits(partial sum of rank r for token t, tensor w
// (0 = Q, 1 = K)).  A word counts as arrived when its epoch field equals the
// call's epoch, so buffers are never cleared between calls: each call on the
// same buffers uses a new epoch (buffers start zeroed, epoch 0 is never used).
// After the exchange words comes one 16-byte trailer whose first word is the
// buffer's abort word: the epoch of the last call in which a wait of this
// rank ran out.
// Each word validates itself and carries the only data exchanged, so the two
// words of a token are written with one relaxed 16-byte store and polled with
// relaxed loads: no fence or release/acquire pair on the exchange path.
// Every wait is bounded by the global timer; on expiry the kernel records a
// code, marks the epoch aborted in the abort word of every rank the launch
// runs so every other wait of the call gives up at once (recording the code
// too), and skips the affected tokens (their outputs are not written).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {
namespace tp {

constexpr int kMaxRanks = 8;     // ranks per tensor-parallel group
constexpr int kMaxLocal = 8;     // ranks one launch may run

struct RankPtrs {
    const char *q_in;
    char *q_out;
    const char *gamma_q;    // this rank's slice of gamma_q
    const char *k_in;
    char *k_out;
    const char *gamma_k;
};

struct TpParams {
    RankPtrs local[kMaxLocal];            // the ranks this launch runs
    unsigned long long *recv[kMaxRanks];  // rank i's receive buffer [R][T][2] + abort word (peer-mapped when remote)
    int64_t q_stride_bytes, k_stride_bytes;
    int64_t T;
    int32_t R;                            // ranks in the group
    int32_t first_rank;                   // rank of local[0]; local[j] is rank first_rank + j
    int32_t n_local;
    int32_t blocks_per_rank;              // G
    int32_t q_vecs, k_vecs;               // 16-byte vectors per shard row
    float inv_hq, inv_hk;                 // fl(1 / Hq_full), fl(1 / Hk_full)
    float eps;
    uint32_t epoch;
    uint64_t timeout_ns;
};

// Host side (qknorm_tp.cu): launch `p` on `stream` with `threads` threads per
// block (128: four warps, one token each) for element type `dtype` (1 = bf16,
// 2 = fp16, 0 = fp32, 3 = E4M3); nv < 0 selects the kernel with NVQ vectors
// per lane for Q and NVK for K, nv = -(8 NVQ + NVK), nv == 0 the kernel for
// rows of any width.  gpu_scope selects the exchange at GPU scope (valid only
// when every rank of the group runs in this launch), else system scope (peer
// memory).  Cooperative when n_local > 1.
cudaError_t launch_tp(const TpParams &p, int dtype, int nv, int threads, bool gpu_scope, cudaStream_t stream,
                      const char **what);

// Blocks of the kernel for (dtype, nv, threads, scope) resident per SM.
cudaError_t tp_blocks_per_sm(int dtype, int nv, int threads, bool gpu_scope, int *out);

// The code a timed-out wait recorded (0 = none); synchronizes the device and
// clears it.
cudaError_t tp_read_and_clear_timeout(int *code);

}  // namespace tp
}  // namespace qkn
