/*
 * qknorm.h — C-ABI of libqknorm.so: layerwise QK-RMSNorm for NVIDIA B200 (sm_100a).
 *
 * What it computes ("SwiftQK: Fast and Communication-Efficient Tensor
 * Parallelism for Query-Key Normalization", arXiv 2608.09160):
 *
 *   Background, RMS-Norm (Equation 1).  For the full projected Q row and the
 *   full projected K row of every token, one factor per row:
 *       S = sum_j x_j^2,   r = 1 / sqrt(S / H + eps),   y_j = (x_j * gamma_j) * r
 *   with eps inside the square root and the mean over the full width H.  (The
 *   page lost the typeset equation; this is the reading its surrounding text,
 *   its RMSNorm citation and the phase descriptions support.)
 *
 *   Phase A.  The factor needs only the squared sum; a hidden-dimension shard
 *   contributes its local squared sum, and the shard sums (fp32) add up to the
 *   global one, with the same semantics as the unsharded form.
 *
 *   Phase B.  The weight multiplication x * gamma does not depend on the
 *   reduction; the global factor r is applied to it and only the final
 *   normalized values are written.
 *
 * Paper, Evaluation, Fig. 2(b): BF16 and FP8-E4M3 activations, FP32
 * accumulation.
 *
 * Arithmetic: elements are widened to fp32; squared sums, the factor and the
 * scaling are fp32 (squares accumulated with fused multiply-add); the mean is
 * formed as S * fl(1/H), with 1/H rounded to fp32 once on the host (exact when
 * H is a power of two); the factor uses the device's rsqrtf; outputs are
 * rounded once to the element type (round-to-nearest-even).  NaN/Inf inputs propagate as IEEE arithmetic does; a
 * squared sum above FLT_MAX overflows to +inf (fp32 accumulation).
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers of the current CUDA device; the caller owns
 *     every buffer.  The library allocates nothing and keeps no state besides a
 *     per-device cache of launch occupancy and a per-thread error message.
 *   - Layout: row-major.  Element (t, j) of a tensor with row stride `stride`
 *     (in ELEMENTS, >= the row width) is at base[t * stride + j].  Packed
 *     [Q | K | V] rows are addressed by passing base and base + Hq with the
 *     packed stride; columns outside [0, width) (V, padding) are never read
 *     or written.
 *   - gamma vectors are contiguous, one per tensor (or per shard, for the
 *     shard entry points), of the element type -- bfloat16 for E4M3 data.
 *   - out == in (same base, same stride) normalizes in place.  Any other
 *     overlap between a written region and any other region is rejected with
 *     QKN_ERR_INVALID_ARG.  Two strided regions with different strides whose
 *     address ranges intersect are rejected even if their elements happen to
 *     be disjoint.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work: it is asynchronous and never synchronizes.
 *   - T == 0 returns QKN_OK without launching anything.
 *   - Arguments are validated on the host before any launch; a rejected call
 *     enqueues nothing.  QKN_ERR_CUDA reports a launch failure (the message
 *     is available from qknorm_last_error on the calling thread).
 *   - Alignment is never an error: when every base pointer and every row
 *     stride in bytes is a multiple of 16, rows move as 16-byte vectors;
 *     otherwise a scalar-access kernel runs (still on the GPU).
 *   - Thread safety: calls may be made from several host threads at once.
 */
#ifndef QKNORM_H
#define QKNORM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QKN_F32 = 0,      /* IEEE binary32 elements; gamma binary32 */
    QKN_BF16 = 1,     /* bfloat16 elements; gamma bfloat16 */
    QKN_F16 = 2,      /* IEEE binary16 elements; gamma binary16 */
    QKN_FP8_E4M3 = 3  /* FP8 E4M3 ("fn": no infinities, largest finite 448)
                         elements; gamma bfloat16.  Outputs round to nearest
                         even and saturate to +-448. */
} qkn_dtype;

typedef enum {
    QKN_OK = 0,
    QKN_ERR_INVALID_ARG = 1,   /* bad size, stride, eps, dtype, null pointer or overlap */
    QKN_ERR_MISALIGNED = 2,    /* reserved: never returned -- unaligned buffers take a
                                  scalar-access kernel instead (see Alignment above) */
    QKN_ERR_UNSUPPORTED = 3,   /* a shape or launch the library cannot run */
    QKN_ERR_CUDA = 4           /* the CUDA runtime reported an error */
} qkn_status;

/*
 * Fused layerwise QK-Norm: normalizes the Q row and the K row of all T tokens
 * in ONE kernel launch (Background, Equation 1; Phase B's fused weight
 * multiplication and store).
 *   q_in, q_out : [T rows, stride q_stride] elements; Q width Hq.
 *   k_in, k_out : [T rows, stride k_stride] elements; K width Hk.
 *   gamma_q [Hq], gamma_k [Hk].
 *   eps >= 0 and finite.  dtype: element type of every buffer.
 * Errors: QKN_ERR_INVALID_ARG for T < 0, Hq or Hk <= 0, a stride below its
 * width, a bad eps or dtype, a null pointer with T > 0, or a forbidden overlap.
 */
qkn_status qknorm_layerwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                            const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                            int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype,
                            void *stream);

/*
 * Phase A, local step, for one hidden-dimension shard of Q and of K: writes
 * the fp32 squared sum of each token's shard row.
 *   q_shard : [T rows, stride q_stride], shard width hq_shard; q_sumsq : [T] fp32 (written).
 *   k_shard : [T rows, stride k_stride], shard width hk_shard; k_sumsq : [T] fp32 (written).
 * For P shards the caller keeps a [P][T] fp32 array per tensor and passes
 * sumsq_all + p * T for shard p.
 * Errors: as qknorm_layerwise; the two sum arrays must not overlap each other
 * or the inputs.
 */
qkn_status qknorm_partial_stats(const void *q_shard, int64_t q_stride, int32_t hq_shard, float *q_sumsq,
                                const void *k_shard, int64_t k_stride, int32_t hk_shard, float *k_sumsq,
                                int64_t T, qkn_dtype dtype, void *stream);

/*
 * Phase A aggregation followed by Phase B for one shard: for each token the P
 * partial sums sumsq_all[p * T + t] are added in fp32 in the fixed order
 * p = 0..P-1, r = 1 / sqrt(S / H_full + eps) divides by the FULL width
 * (Hq_full / Hk_full, not the shard width), and the shard's elements are
 * written as (x * gamma_shard) * r.
 *   q_in, q_out : [T rows, stride q_stride], width hq_shard; gamma_q_shard [hq_shard].
 *   q_sumsq_all : [P][T] fp32, contiguous.   Hq_full >= hq_shard.
 *   (same for K.)   P >= 1.
 * Errors: as qknorm_layerwise, plus P < 1 or a full width below its shard
 * width; outputs must not overlap the sum arrays.
 */
qkn_status qknorm_combine_apply(const void *q_in, void *q_out, const void *gamma_q_shard, int64_t q_stride,
                                int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full,
                                const void *k_in, void *k_out, const void *gamma_k_shard, int64_t k_stride,
                                int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full,
                                int32_t P, int64_t T, float eps, qkn_dtype dtype, void *stream);

/*
 * Multi-shard forms of the two calls above, for P hidden-dimension shards of Q
 * and of K held in separate buffers on this GPU (Phase A: every shard's local
 * squared sum; its aggregation in the fixed order p = 0..P-1; Phase B: each
 * shard scaled by the global factor).  Each covers all P shards in ONE kernel
 * launch instead of P, with the same results as the per-shard calls:
 *   qknorm_partial_stats_shards  ==  for p in 0..P-1:
 *       qknorm_partial_stats(q_shards[p], ..., q_sumsq_all + p * T,
 *                            k_shards[p], ..., k_sumsq_all + p * T, ...)
 *   qknorm_combine_apply_shards  ==  for p in 0..P-1:
 *       qknorm_combine_apply(q_in[p], q_out[p], gamma_q_shards[p], ..., q_sumsq_all, Hq_full,
 *                            k_in[p], k_out[p], gamma_k_shards[p], ..., k_sumsq_all, Hk_full, P, ...)
 * (a squared sum may differ in its last bit from the per-shard call's where
 * the two launches group the shard's row differently; both are within the
 * parity tolerances).
 *   P in [1, 8].  Every Q shard has width hq_shard and row stride q_stride;
 *   likewise for K.  q_sumsq_all / k_sumsq_all: [P][T] fp32, contiguous.
 *   q_out[p] == q_in[p] normalizes shard p in place.
 * Errors: as the per-shard calls, plus P outside [1, 8]; no output may
 * overlap any other shard's operands.  When the rows cannot move as 16-byte
 * vectors (unaligned) or are wider than 32 KB, the call runs shard by shard.
 */
qkn_status qknorm_partial_stats_shards(int32_t P, const void *const *q_shards, int64_t q_stride, int32_t hq_shard,
                                       float *q_sumsq_all, const void *const *k_shards, int64_t k_stride,
                                       int32_t hk_shard, float *k_sumsq_all, int64_t T, qkn_dtype dtype,
                                       void *stream);
qkn_status qknorm_combine_apply_shards(int32_t P, const void *const *q_in, void *const *q_out,
                                       const void *const *gamma_q_shards, int64_t q_stride, int32_t hq_shard,
                                       const float *q_sumsq_all, int32_t Hq_full, const void *const *k_in,
                                       void *const *k_out, const void *const *gamma_k_shards, int64_t k_stride,
                                       int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full, int64_t T,
                                       float eps, qkn_dtype dtype, void *stream);

/*
 * Fused layerwise QK-Norm of rows held in HOST memory, end to end: the T
 * tokens flow in chunks of chunk_tokens through a ring of device buffers, and
 * for each chunk the Q and K rows are copied host->device, normalized in
 * place on the device by the same kernel as qknorm_layerwise (Background,
 * Equation 1; Phase B), and copied device->host.  The host->device copy of
 * one chunk, the kernel on the previous one and the device->host copy of the
 * one before that overlap on three streams.
 *   q_in, q_out, k_in, k_out : HOST pointers, rows as in qknorm_layerwise
 *       ([T rows, stride q_stride] / [T rows, stride k_stride] elements).
 *       Page-locked memory (cudaHostAlloc / cudaHostRegister) lets the copies
 *       run asynchronously at full speed; pageable memory works but the copies
 *       then stage through the driver.  out == in normalizes in place; for
 *       packed [Q | K | V] host rows pass base and base + Hq with the packed
 *       stride: only the Q and K columns travel, V is neither read nor written.
 *   gamma_q [Hq], gamma_k [Hk] : DEVICE pointers (resident weights).
 *   ring : DEVICE buffer owned by the caller, 256-byte aligned, of ring_bytes
 *       bytes; it holds floor(ring_bytes / slot) slots (at most
 *       QKN_HOST_MAX_SLOTS), a slot being chunk_tokens rows of Q then of K.
 *       qknorm_layerwise_host_ring_bytes gives the size for a slot count; two
 *       slots overlap copies in both directions with the kernel, three also
 *       let a copy-in run ahead.
 *   stream : the call's stream -- the kernels run on it, the copies start
 *       after everything queued on it before the call, and the call is
 *       complete (every output row back in host memory) once `stream`
 *       reaches the point where the call returns.  copy_in_stream and
 *       copy_out_stream carry the two copy directions; three different
 *       streams give the overlap (equal streams are correct, only serial).
 *       Calls that share a ring must be ordered through `stream`.
 * Host memory must stay valid and unmodified until the call is complete.
 * Errors: as qknorm_layerwise (arguments validated before anything is
 * enqueued; host regions checked for overlap by address), plus
 * QKN_ERR_INVALID_ARG for chunk_tokens < 1, a null or unaligned ring, a ring
 * smaller than one slot, or a ring overlapping gamma.  A QKN_ERR_CUDA from a
 * failed copy or launch may leave earlier chunks enqueued.
 * No paper counterpart beyond the kernel: this is the library's end-to-end
 * path for callers whose activations live in host memory.
 */
#define QKN_HOST_MAX_SLOTS 8
qkn_status qknorm_layerwise_host(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                 const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                 int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype, void *ring,
                                 int64_t ring_bytes, int64_t chunk_tokens, void *stream, void *copy_in_stream,
                                 void *copy_out_stream);

/* Bytes of a ring of `slots` slots for qknorm_layerwise_host: slots *
 * (round_up(chunk_tokens * Hq * esz, 256) + round_up(chunk_tokens * Hk * esz,
 * 256)), esz the element size; -1 for chunk_tokens < 1 or > 2^31, Hq or Hk <
 * 1, slots outside [1, QKN_HOST_MAX_SLOTS] or an unknown dtype. */
int64_t qknorm_layerwise_host_ring_bytes(int64_t chunk_tokens, int32_t Hq, int32_t Hk, qkn_dtype dtype,
                                         int32_t slots);

/*
 * Headwise QK-Norm (Background: the other granularity, "an independent factor
 * for each attention head"): token t's Q row holds q_heads heads of head_dim
 * elements, head h at columns [h * head_dim, (h + 1) * head_dim); K likewise
 * with k_heads heads.  Each head is normalized on its own:
 *       S = sum_j x_j^2 over the head,  r = 1 / sqrt(S / head_dim + eps),
 *       y_j = (x_j * gamma_j) * r,
 * with gamma_q [head_dim] shared by all Q heads and gamma_k [head_dim] by all K
 * heads.  ONE launch for Q and K.  Strides as in qknorm_layerwise (stride >=
 * heads * head_dim); out == in normalizes in place.  Heads move as 16-byte
 * vectors when head_dim * element size is a multiple of 16 (and the usual
 * pointer/stride alignment holds).  Under tensor parallelism whole heads live
 * on one rank, so the headwise form needs no cross-shard statistics.
 * Errors: as qknorm_layerwise, plus q_heads, k_heads or head_dim <= 0, or
 * T * heads >= 2^31.
 */
qkn_status qknorm_headwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride, int32_t q_heads,
                           const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride, int32_t k_heads,
                           int64_t T, int32_t head_dim, float eps, qkn_dtype dtype, void *stream);

/*
 * QKV projection with Phase A's partial sums in the GEMM epilogue (Background:
 * in a Pre-LN layer linear projections of the hidden state produce Q, K and V,
 * and QK-Norm sits between the Q/K projections and attention; Phase A: the
 * RMS factor needs only each shard's squared sum).  Runs on the tensor cores
 * (tcgen05, bf16 operands, fp32 accumulation).
 *   x   : [T rows, stride x_stride] bfloat16, the hidden states, width D.
 *   w   : [N rows, stride w_stride] bfloat16, N = Hq + Hk + Hv, one row per
 *         output column (the linear layer's weight as stored): Q columns
 *         first, then K, then V.
 *   qkv : [T rows, stride qkv_stride] bfloat16 output,
 *         qkv[t][n] = RNE_bf16( sum_d x[t][d] * w[n][d] ).
 *   q_sumsq_all : [Hq / 256][T] fp32; entry [p][t] is the squared sum of the
 *         stored (rounded) values qkv[t][256p .. 256p + 255], summed in column
 *         order.  k_sumsq_all likewise for the K columns, [Hk / 256][T].
 * These are exactly the inputs qknorm_combine_apply expects with 256-column
 * shards; qknorm_qkv_projection below runs both steps.
 * Requirements: dtype QKN_BF16 (else QKN_ERR_UNSUPPORTED); Hq, Hk > 0 and Hv
 * >= 0 multiples of 256 (else QKN_ERR_UNSUPPORTED); D >= 1 (any D: the k
 * loop reads zeros past it); x, w, qkv 16-byte aligned with strides a
 * multiple of 8 elements; T < 2^31; qkv must not overlap x, w or the sums.
 * Asynchronous on `stream`; allocates nothing.  T = 0 is a no-op.
 */
qkn_status qknorm_qkv_gemm_stats(const void *x, int64_t x_stride, const void *w, int64_t w_stride, void *qkv,
                                 int64_t qkv_stride, int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv,
                                 float *q_sumsq_all, float *k_sumsq_all, qkn_dtype dtype, void *stream);

/* Bytes of workspace qknorm_qkv_projection needs: (Hq/256 + Hk/256) * T * 4,
 * or -1 when the sizes are invalid. */
int64_t qknorm_qkv_projection_workspace_bytes(int64_t T, int32_t Hq, int32_t Hk);

/*
 * Projection followed by layerwise QK-Norm of its Q and K columns, two
 * launches on `stream`: qknorm_qkv_gemm_stats writing the partial sums into
 * `workspace`, then Phase A's aggregation (partials added in order p = 0, 1,
 * ..., fp32) and Phase B's scaling of the Q and K columns of qkv in place:
 *   r = 1 / sqrt(S / H + eps),  qkv[t][j] = RNE_bf16( (qkv[t][j] * gamma_j) * r )
 * with H = Hq for the Q columns (gamma_q [Hq]) and Hk for the K columns
 * (gamma_k [Hk]); V columns keep the projection.  The caller owns
 * `workspace` (>= qknorm_qkv_projection_workspace_bytes, 4-byte aligned); its
 * contents on return are the partial sums.  Same requirements and errors as
 * qknorm_qkv_gemm_stats, plus eps finite and >= 0 and non-null gamma.
 */
qkn_status qknorm_qkv_projection(const void *x, int64_t x_stride, const void *w, int64_t w_stride, void *qkv,
                                 int64_t qkv_stride, const void *gamma_q, const void *gamma_k, int64_t T, int32_t D,
                                 int32_t Hq, int32_t Hk, int32_t Hv, float eps, void *workspace,
                                 int64_t workspace_bytes, qkn_dtype dtype, void *stream);

/*
 * qknorm_qkv_projection for callers that cannot allocate device memory: a
 * host engine that owns every device allocation and forbids new ones once it
 * is serving, or a latency-critical path on which a cudaMalloc (which may
 * synchronize the device) is not acceptable.  Same arguments, results and
 * errors as qknorm_qkv_projection, without the workspace: the partial sums go
 * to a 4 MiB array built into this library (qknorm_qkv_projection_noalloc_max_bytes),
 * which every GPU that loads the library holds until the process exits.
 * Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library
 * call.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  The address is kept with the id of the context
 * it belongs to and looked up again when the calling thread's context is
 * another one (after cudaDeviceReset, say): the first call after such a
 * change should also come before any capture.
 * Limits: the call's workspace, qknorm_qkv_projection_workspace_bytes(T, Hq,
 * Hk) = (Hq/256 + Hk/256) * T * 4 bytes, must fit in the 4 MiB (e.g. T up to
 * 32768 with Hq = Hk = 4096); larger calls return QKN_ERR_INVALID_ARG before
 * any launch.
 * Sharing: all calls on a device use the same array, and it keeps the last
 * call's contents.  Each call writes every partial sum before reading it;
 * but two calls that can run at the same time on the GPU (different streams
 * without ordering between them, or different host threads) race on the
 * array and may corrupt each other's results.  Order such calls on one
 * stream or with events.
 * The paper has no counterpart: this is a deployment variant of this library.
 */
qkn_status qknorm_qkv_projection_noalloc(const void *x, int64_t x_stride, const void *w, int64_t w_stride,
                                         void *qkv, int64_t qkv_stride, const void *gamma_q, const void *gamma_k,
                                         int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, float eps,
                                         qkn_dtype dtype, void *stream);

/* Bytes of the built-in scratch qknorm_qkv_projection_noalloc uses (4 MiB). */
int64_t qknorm_qkv_projection_noalloc_max_bytes(void);

/*
 * Tensor-parallel layerwise QK-Norm: the paper's multi-GPU kernel (Phase A:
 * each rank squares and sums its hidden-dimension shard and the ranks add
 * their scalar partial sums in fp32; Phase B: the global factor scales the
 * shard times gamma; deadlock-safe persistent blocks).  One warp carries a
 * token, publishing two tokens ahead of the one it finishes so that the
 * exchange overlaps the loads of later tokens.
 *   R ranks each hold a shard of every token's Q row (hq_shard columns of
 *   Hq_full) and K row (hk_shard of Hk_full).  This call runs the n_local
 *   ranks first_rank .. first_rank + n_local - 1; local rank j's rows are
 *   q_in[j] / q_out[j] ([T rows, stride q_stride]), gamma slice gamma_q[j]
 *   [hq_shard], and likewise for K.  out == in normalizes in place.
 *   recv[r] (r < R) is rank r's receive buffer, qknorm_tp_recv_bytes(R, T)
 *   bytes, 16-byte aligned: a device pointer valid on this GPU -- its own
 *   memory for local ranks, a peer mapping (cudaIpcOpenMemHandle or similar)
 *   for ranks on other GPUs.  A buffer holds R * T pairs of 64-bit exchange
 *   words and a 16-byte trailer (its abort word).  Buffers start zeroed and
 *   are never cleared by the library; each call on the same buffers passes a
 *   new epoch (> 0), and all ranks of one call pass the same epoch.
 *   Result: y = (x * gamma) * r with r = 1 / sqrt(S / H_full + eps) and S the
 *   ranks' partial sums added in rank order 0 .. R-1, identical on every rank.
 * Deployments: one GPU per rank (n_local = 1, each GPU calls with its own
 * rank; pass the same blocks_per_rank on every rank, or 0 on identical GPUs),
 * or several ranks in one call on one GPU (their blocks wait on one another,
 * so the launch is cooperative and must fit on the GPU at once).
 * Waits are bounded by timeout_ns (0 = 2 s); one that runs out reports code 4
 * through qknorm_device_timeouts and writes the call's epoch into the abort
 * word of every rank the call runs; every other wait of that call on those
 * buffers then gives up and reports code 4 as well, and the tokens concerned
 * are left unwritten.  The abort belongs to those buffers and that epoch:
 * later epochs, and other buffers, are not affected.
 * Requirements: 1 <= R <= 8, n_local <= 8; dtype any of qkn_dtype; 16-byte
 * aligned buffers and shard widths / strides that are whole 16-byte vectors
 * (else QKN_ERR_UNSUPPORTED); no output overlapping another operand, and no
 * receive buffer overlapping another or any local rank's rows or gamma
 * (else QKN_ERR_INVALID_ARG).  T = 0 is a no-op.  Asynchronous on `stream`;
 * allocates nothing.
 */
/* Bytes of one receive buffer: R * T * 16 + 16; -1 for R outside [1, 8],
 * T < 0 or T >= 2^31. */
int64_t qknorm_tp_recv_bytes(int32_t R, int64_t T);
qkn_status qknorm_tp_layerwise(int32_t R, int32_t first_rank, int32_t n_local, const void *const *q_in,
                               void *const *q_out, const void *const *gamma_q, int64_t q_stride, int32_t hq_shard,
                               int32_t Hq_full, const void *const *k_in, void *const *k_out,
                               const void *const *gamma_k, int64_t k_stride, int32_t hk_shard, int32_t Hk_full,
                               int64_t T, float eps, qkn_dtype dtype, void *const *recv, uint32_t epoch,
                               int32_t blocks_per_rank, uint64_t timeout_ns, void *stream);

/*
 * Every wait inside the projection kernel is bounded (2 s); one that runs out
 * records a non-zero code (1 = TMA producer, 2 = MMA issuer, 3 = epilogue;
 * 4 = a tensor-parallel exchange wait) and the kernel returns early with its
 * output incomplete.  This call
 * synchronizes the current device, stores that code in *code (0 = none) and
 * clears it.  No paper counterpart: a safety check of this library.
 */
qkn_status qknorm_device_timeouts(int32_t *code);

/* Short English name of a status code (static storage). */
const char *qknorm_status_string(qkn_status s);

/* Message describing the last non-OK status returned on the calling thread
 * ("" if none).  The pointer stays valid until the thread's next call. */
const char *qknorm_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int qknorm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKNORM_H */
