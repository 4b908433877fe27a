/*
 * qknorm_plan.h — launch planning for libqknorm.so, exported so that the host
 * logic can be tested without a GPU and so that a caller can pin a launch
 * shape (benchmark sweeps, per-variant tests).  Include after qknorm.h.
 *
 * Execution model (the single-GPU form of the paper's "deadlock-safe
 * persistent execution"): a kernel launches a bounded grid and each CTA loops
 * over items blockIdx.x, blockIdx.x + grid, ...  An item is a group of rows
 * of one tensor (a CTA of `threads` threads holds threads / group rows); the
 * items of the Q rows come first, then those of the K rows, so every CTA
 * gets a near-equal share of each tensor's rows whatever the grid.  The
 * planner launches as many CTAs as can be resident at once, except where a
 * fused launch has at least 4 items per resident slot -- then 3 (below 6
 * items per slot) or 4 CTAs per slot, so that the hardware hands the
 * remaining items to the CTAs that finish first -- and the combine/apply
 * pass over rows of 129..160 vectors, which also runs 4 per slot.  No CTA
 * ever waits on another, so any grid is safe.
 *
 * Kernel kinds:
 *   QKN_KERNEL_REGISTER  one pass; the row (or head) is held in registers by
 *                        a group of threads -- 1, 2, 4, 8 or 16 lanes, or a
 *                        multiple of 32 dividing the CTA, the smallest that
 *                        covers the row with vec_per_thread 16-byte vectors
 *                        each; lane l owns vectors l, l + group, ... of every
 *                        row, so it keeps its gamma vectors in registers across
 *                        the rows of one tensor; every element is read once and
 *                        written once.
 *                        Needs 16-byte alignment (see qknorm.h) and a row of
 *                        at most vec_per_thread * threads vectors.
 *   QKN_KERNEL_TWOPASS_VEC  two passes over the row with 16-byte vectors
 *                        (the second pass re-reads x, mostly from L2); for
 *                        rows too wide for registers.
 *   QKN_KERNEL_TWOPASS_SCALAR  two passes with element-wise access; for
 *                        buffers that are not 16-byte aligned.
 */
#ifndef QKNORM_PLAN_H
#define QKNORM_PLAN_H

#include <stdint.h>
#include "qknorm.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QKN_KERNEL_REGISTER = 0,
    QKN_KERNEL_TWOPASS_VEC = 1,
    QKN_KERNEL_TWOPASS_SCALAR = 2
} qkn_kernel_kind;

typedef struct {
    int32_t kernel;          /* qkn_kernel_kind */
    int32_t vec_per_thread;  /* QKN_KERNEL_REGISTER only: 1, 2, 4 or 8; also 5 for the
                                partial-sum and combine/apply passes (one warp per row
                                of 129..160 vectors) */
    int32_t threads;         /* threads per CTA: a multiple of 32 in [32, 1024] */
    int64_t grid;            /* number of CTAs, >= 1 */
} qkn_launch;

/* Largest CTA the register kernel accepts for a given vec_per_thread
 * (1024 for 1 and 2, 512 for 4, 256 for 5 and 8); 0 for an unsupported
 * value.  5 exists for the partial-sum and combine/apply passes only. */
int32_t qknorm_register_max_threads(int32_t vec_per_thread);

/*
 * Chooses kernel kind, vec_per_thread and threads (grid is left 0) from:
 *   rows       : row items in the launch (2 * T),
 *   units_max  : the widest row, in 16-byte vectors if `vectorized`, else in elements,
 *   vectorized : 1 if every pointer and row stride is 16-byte aligned,
 *   sm_count   : streaming multiprocessors on the device,
 *   elem_bytes : bytes per element of x (4, 2 or 1).
 * Pure function of its arguments; needs no GPU.  QKN_ERR_INVALID_ARG for
 * rows < 1, units_max < 1, sm_count < 1 or another elem_bytes.
 */
qkn_status qknorm_plan_shape(int64_t rows, int64_t units_max, int32_t vectorized, int32_t sm_count,
                             int32_t elem_bytes, qkn_launch *out);

/*
 * CTAs for `rows` items when `blocks_per_sm` CTAs fit on each of `sm_count`
 * SMs: min(rows, blocks_per_sm * sm_count), i.e. every resident slot is
 * filled and no CTA waits for a slot.  Pure; returns 0 for rows < 1, and
 * treats a non-positive blocks_per_sm or sm_count as 1.
 */
int64_t qknorm_plan_grid(int64_t rows, int32_t blocks_per_sm, int32_t sm_count);

/*
 * 1 if two row sets may share a byte, 0 if they are provably disjoint.  A row
 * set is `rows` byte ranges [base + t * stride, base + t * stride + width).
 * Exact when either set has one row or both strides are equal; otherwise any
 * intersection of the address ranges counts as overlap (conservative).
 * Empty sets (rows < 1 or width < 1) never overlap.
 */
int qknorm_regions_overlap(uint64_t a_base, int64_t a_width, int64_t a_stride, int64_t a_rows,
                           uint64_t b_base, int64_t b_width, int64_t b_stride, int64_t b_rows);

/*
 * The launch qknorm_layerwise would use for these arguments on the current
 * device (queries the SM count and the kernel's occupancy; needs a GPU).
 * Validates its arguments exactly as qknorm_layerwise does.
 */
qkn_status qknorm_layerwise_plan(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                 const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                 int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype,
                                 qkn_launch *out);

/*
 * qknorm_layerwise with a caller-chosen launch.  The squared sum is formed in
 * an order fixed by the launch shape (per-thread sequential, then a warp
 * butterfly, then warp partials in order), so a given shape is deterministic
 * run to run, while two shapes may differ in the last bits of the sum and
 * hence by one unit in the last place of an output.  Beyond the checks of
 * qknorm_layerwise, QKN_ERR_INVALID_ARG when: threads is not a multiple of 32
 * in [32, 1024]; grid < 1 or grid > 2^31 - 1; a vector kernel is asked for on
 * unaligned buffers; for the register kernel, vec_per_thread is not 1, 2, 4
 * or 8, threads exceeds qknorm_register_max_threads(vec_per_thread), or the
 * widest row has more than vec_per_thread * threads vectors.
 */
qkn_status qknorm_layerwise_launch(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                   const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                   int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype,
                                   void *stream, const qkn_launch *launch);

/* qknorm_headwise with a caller-chosen launch (rows are heads). */
qkn_status qknorm_headwise_launch(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                  int32_t q_heads, const void *k_in, void *k_out, const void *gamma_k,
                                  int64_t k_stride, int32_t k_heads, int64_t T, int32_t head_dim, float eps,
                                  qkn_dtype dtype, void *stream, const qkn_launch *launch);

/*
 * qknorm_partial_stats / qknorm_combine_apply with a caller-chosen launch;
 * the same launch rules and checks as qknorm_layerwise_launch apply.
 */
qkn_status qknorm_partial_stats_launch(const void *q_shard, int64_t q_stride, int32_t hq_shard, float *q_sumsq,
                                       const void *k_shard, int64_t k_stride, int32_t hk_shard, float *k_sumsq,
                                       int64_t T, qkn_dtype dtype, void *stream, const qkn_launch *launch);

qkn_status qknorm_combine_apply_launch(const void *q_in, void *q_out, const void *gamma_q_shard, int64_t q_stride,
                                       int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full,
                                       const void *k_in, void *k_out, const void *gamma_k_shard, int64_t k_stride,
                                       int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full,
                                       int32_t P, int64_t T, float eps, qkn_dtype dtype, void *stream,
                                       const qkn_launch *launch);

/*
 * qknorm_partial_stats_shards / qknorm_combine_apply_shards with a
 * caller-chosen launch of the register kernel (the launch rules and checks of
 * qknorm_layerwise_launch, with the widest shard row as the row); the shard
 * rows must be 16-byte aligned and at most 32 KB, else QKN_ERR_INVALID_ARG.
 */
qkn_status qknorm_partial_stats_shards_launch(int32_t P, const void *const *q_shards, int64_t q_stride,
                                              int32_t hq_shard, float *q_sumsq_all, const void *const *k_shards,
                                              int64_t k_stride, int32_t hk_shard, float *k_sumsq_all, int64_t T,
                                              qkn_dtype dtype, void *stream, const qkn_launch *launch);
qkn_status qknorm_combine_apply_shards_launch(int32_t P, const void *const *q_in, void *const *q_out,
                                              const void *const *gamma_q_shards, int64_t q_stride, int32_t hq_shard,
                                              const float *q_sumsq_all, int32_t Hq_full, const void *const *k_in,
                                              void *const *k_out, const void *const *gamma_k_shards,
                                              int64_t k_stride, int32_t hk_shard, const float *k_sumsq_all,
                                              int32_t Hk_full, int64_t T, float eps, qkn_dtype dtype, void *stream,
                                              const qkn_launch *launch);

/*
 * qknorm_tp_layerwise with the memory scope of the exchange chosen by the
 * caller.  scope 0: as qknorm_tp_layerwise (GPU-scope loads and stores when
 * every rank of the group runs in this call, system scope otherwise); scope
 * 1: system scope always -- the instantiation a one-rank-per-GPU deployment
 * runs over peer memory -- so that it can be checked with every rank in one
 * call on one GPU.  Same arguments, results and errors as
 * qknorm_tp_layerwise, plus QKN_ERR_INVALID_ARG for another scope.
 */
qkn_status qknorm_tp_layerwise_scope(int32_t R, int32_t first_rank, int32_t n_local, const void *const *q_in,
                                     void *const *q_out, const void *const *gamma_q, int64_t q_stride,
                                     int32_t hq_shard, int32_t Hq_full, const void *const *k_in, void *const *k_out,
                                     const void *const *gamma_k, int64_t k_stride, int32_t hk_shard, int32_t Hk_full,
                                     int64_t T, float eps, qkn_dtype dtype, void *const *recv, uint32_t epoch,
                                     int32_t blocks_per_rank, uint64_t timeout_ns, int32_t scope, void *stream);

/*
 * The schedule of the projection GEMM (qknorm_qkv_gemm_stats and the
 * projection entry points; the QKV projection of the SwiftQK paper's
 * Background section, with Phase A's partial sums in its epilogue).  A unit
 * is one tensor-core tile of 256 tokens x 256 output columns; persistent CTA
 * pairs take units c, c + clusters, ... in a grouped raster: within a group
 * of group_units token blocks the token block runs fastest, then the column
 * tile, then the group.  The group is sized by what fits in half of L2: all
 * token blocks when X fits, one when W fits, else about sqrt(clusters).
 */
typedef struct {
    int32_t clusters;    /* CTA groups launched: min(units, resident groups) */
    int32_t units;       /* work units: ceil(T / 256) * (Hq + Hk + Hv) / 256 */
    int32_t group_units; /* token blocks (of 256 tokens) per raster group */
} qkn_gemm_schedule;

/*
 * The schedule for `clusters` resident CTA groups on a GPU with an L2 of
 * `l2_bytes` bytes.  Pure function of its arguments; needs no GPU.
 * QKN_ERR_INVALID_ARG for a null `out`, T outside [1, 2^31), D < 1, Hq < 1,
 * Hk < 1, Hv < 0, clusters < 1 or l2_bytes < 0; QKN_ERR_UNSUPPORTED when Hq,
 * Hk or Hv is not a multiple of 256 or the output has more than 2^30 tiles.
 */
qkn_status qknorm_qkv_gemm_schedule(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, int32_t clusters,
                                    int64_t l2_bytes, qkn_gemm_schedule *out);

/*
 * The schedule the projection entry points use for this shape on the
 * current device (queries the resident CTA pairs and the L2 size; needs a
 * GPU).  Errors as qknorm_qkv_gemm_schedule, plus QKN_ERR_CUDA when a query
 * fails.
 */
qkn_status qknorm_qkv_gemm_plan(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, qkn_gemm_schedule *out);

#ifdef __cplusplus
}
#endif

#endif /* QKNORM_PLAN_H */
