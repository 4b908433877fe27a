// QKV projection on the sm_100a tensor cores with Phase A's partial squared
// sums produced in the epilogue.
//
// Method: "SwiftQK: Fast and Communication-Efficient Tensor Parallelism for
// Query-Key Normalization" (arXiv 2608.09160).
//   Background: in a Pre-LN layer linear projections produce Q, K and V, and
//     layerwise QK-Norm normalizes the full projected Q and K rows before
//     attention.
//   Phase A: the RMS factor needs only the squared sum of the row; each
//     hidden-dimension shard contributes the squared sum of its own columns
//     and the partial sums are added in fp32.
// Here a shard is one 256-column output tile of the projection: the epilogue
// that stores the tile's bf16 values also writes, per token, the squared sum
// of those stored values.  The combine / factor / scale steps then run as the
// usual apply pass (Phase A aggregation + Phase B).
//
// Kernel shape: persistent, clusters of kCta CTAs (320 threads each, one per
// SM), as many as are resident at once.  A work unit is one MMA tile of
// 128 * kCta tokens x 256 columns; cluster c takes units c, c + clusters, ...
// in a grouped raster (token block fastest within a group of group_units
// token blocks, then the column tile, then the group; the host sizes the
// group by what fits in L2).  With kCta = 2 the pair's leader issues
// tcgen05.mma cta_group::2 (M = 256) and each CTA receives its 128 rows of
// the 128 x 256 result in its own TMEM.  Roles, per CTA:
//   warp 0, lane 0 : TMA producer.  X tile [128 x 64] and this CTA's half of
//                    the W tile [256 / kCta x 64] per k-block into a kStages
//                    shared-memory ring, 128-byte swizzle, completion counted
//                    on the leader's mbarrier per stage; the ring runs on
//                    across tiles.
//   warp 1         : allocates 512 TMEM columns, two fp32 accumulators of
//                    128 lanes x 256 columns (lane = tile row); in the leader
//                    lane 0 issues the MMAs (K = 16, bf16 in, fp32
//                    accumulate), four per k-block, into the accumulator of
//                    the tile's parity, frees each stage in both CTAs with
//                    tcgen05.commit when its MMAs have read it, and signals
//                    both epilogues when a tile's accumulator is complete.
//   warps 2..9     : epilogue, two warps per TMEM lane quarter.  Warp w
//                    reads TMEM lanes 32*(w%4) .. +31 (one tile row per
//                    thread); warps 2..5 take columns 0..127 of the tile and
//                    warps 6..9 columns 128..255, in 32-column chunks.  Each
//                    value is rounded to bf16 (nearest even) and stored; for
//                    Q and K tiles each half sums the squares of its rounded
//                    values in column order (fp32 fma), and the tile's
//                    partial for the row is (first half) + (second half).
//                    Then the accumulator goes back to the MMA thread.  With
//                    two accumulators the epilogue of one tile overlaps the
//                    MMAs of the next.
// Every mbarrier wait is bounded by the global timer; on expiry the kernel
// records a code in a device word, skips the rest of its work, lets its
// in-flight loads land, frees its TMEM and returns, so the context stays
// usable.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {
namespace gemm {

constexpr int kBM = 128;           // tile rows (tokens) = TMEM lanes
constexpr int kBN = 256;           // tile columns = one partial-sum shard
constexpr int kBK = 64;            // k-block: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;         // K of one tcgen05.mma kind::f16
#ifndef QKN_GEMM_CTA_GROUP
#define QKN_GEMM_CTA_GROUP 2
#endif
// CTAs per MMA: 2 = a cluster of two CTAs on two SMs runs one 256 x 256 tile
// with tcgen05 cta_group::2 (each CTA holds 128 rows of X and 128 rows of W
// per k-block and receives 128 x 256 of the result); 1 = one CTA per 128 x 256
// tile.
constexpr int kCta = QKN_GEMM_CTA_GROUP;
static_assert(kCta == 1 || kCta == 2, "one or two CTAs per MMA");
#ifndef QKN_GEMM_STAGES
#define QKN_GEMM_STAGES 0
#endif
// Shared-memory ring depth: 6 x 32 KB for the pair form, 4 x 48 KB with one
// CTA per tile.  (Measured on a B200: 7 x 32 KB, the most that fits, was 1-2%
// slower than 6 at T = 4096.)
constexpr int kStages = QKN_GEMM_STAGES > 0 ? QKN_GEMM_STAGES : (kCta == 2 ? 6 : 4);
#ifndef QKN_GEMM_EPI_WARPS
#define QKN_GEMM_EPI_WARPS 8
#endif
#ifndef QKN_GEMM_GROUP_M
#define QKN_GEMM_GROUP_M -1
#endif
constexpr int kEpiWarps = QKN_GEMM_EPI_WARPS;  // 4 or 8: one or two per TMEM lane quarter
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "the epilogue has 4 or 8 warps");
constexpr int kEpiSplit = kEpiWarps / 4;       // warps sharing one lane quarter (column split)
constexpr int kEpiCols = kBN / kEpiSplit;      // tile columns per epilogue warp
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kGroupM = QKN_GEMM_GROUP_M;      // token blocks per raster group: -1 = the host's choice, 0 = one group
constexpr int kBNLocal = kBN / kCta;           // W rows (output columns) each CTA stages
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBNLocal * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;    // per CTA and stage
constexpr int kTxBytes = kStageBytes * kCta;      // bytes one full barrier phase counts
constexpr int kAccCols = kBN;      // fp32 columns of one accumulator
constexpr int kTmemCols = 2 * kAccCols;
// ring + barriers (2 * kStages + 4 mbarriers) + TMEM address slot + 1 KB
// alignment slack for the 128-byte-swizzle atoms
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
// the kernel's static shared memory (partial-sum halves, flags) is about
// 1 KB; ring + static must stay within the 227 KB a CTA may use
static_assert(kSmemBytes + 2 * kBM * 4 + 64 <= 232448, "ring + static shared memory within 227 KB");

struct GemmParams {
    char *qkv;               // [T][qkv_stride] bf16, columns [0, N)
    int64_t qkv_stride_bytes;
    float *q_sumsq;          // [Hq / kBN][T] or null
    float *k_sumsq;          // [Hk / kBN][T] or null
    int64_t T;
    int32_t k_blocks;        // ceil(D / kBK)
    int32_t q_tiles;         // Hq / kBN
    int32_t k_tiles;         // Hk / kBN
    int32_t n_tiles;         // N / kBN
    int32_t m_tiles;         // ceil(T / kBM): 128-token tiles
    int32_t m_units;         // ceil(T / (kBM * kCta)): token blocks of one MMA
    int32_t num_units;       // m_units * n_tiles: work units (one per CTA group)
    int32_t group_units;     // token blocks per raster group, 1 .. m_units
    uint64_t timeout_ns;     // bound on every mbarrier wait
};

// Error codes written to the device word when a wait runs out.
enum : int { kErrNone = 0, kErrProducer = 1, kErrMma = 2, kErrEpilogue = 3 };

}  // namespace gemm
}  // namespace qkn

namespace qkn {
namespace gemm {

// Host side (qkv_gemm.cu).  Encodes the TMA maps for X [T][D] (row stride
// x_stride elements) and W [N][D] (row stride w_stride) and launches one CTA
// per output tile on `stream`.  Pointers must be 16-byte aligned and strides
// multiples of 8 elements (the caller checks).  On failure *what names the
// step that failed (static storage).
cudaError_t launch_qkv_gemm(const void *x, int64_t x_stride, const void *w, int64_t w_stride, int32_t D,
                            int32_t N, const GemmParams &p, cudaStream_t stream, const char **what);

// Raster group (pure host function): sets p->group_units from p's tile
// counts for a launch of min(num_units, clusters) CTA groups on a GPU with an
// L2 of l2_bytes.
void schedule_qkv_gemm(GemmParams *p, int32_t D, int32_t N, int clusters, int64_t l2_bytes);

// CTA groups of the kernel resident at once on the current device (cached per
// device); on failure *what names the step that failed.
cudaError_t qkv_gemm_clusters(int *clusters, const char **what);

// The device word a bounded wait writes when it runs out (0 = none); reading
// synchronizes the current device and clears the word.
cudaError_t read_and_clear_timeout(int *code);

}  // namespace gemm
}  // namespace qkn
