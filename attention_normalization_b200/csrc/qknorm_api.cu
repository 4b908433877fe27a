// Host side of libqknorm.so: argument validation, overlap checks, launch
// planning and the extern "C" entry points declared in include/qknorm.h and
// include/qknorm_plan.h.
//
// Every entry point validates on the host before enqueueing anything, so a
// rejected call never reaches the GPU.  Nothing here allocates device memory
// or synchronizes.

#include <cuda.h>  // CUcontext / CUresult types only: driver entry points are fetched at run time
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "qknorm.h"
#include "qknorm_plan.h"
#include "qknorm_kernels.cuh"
#include "qkv_gemm.cuh"
#include "qknorm_tp.cuh"

#ifndef QKNORM_VERSION
#define QKNORM_VERSION 200  // 0.2.0: status codes of the boundary contract (UNSUPPORTED 3, CUDA 4)
#endif

namespace {

// ---------------------------------------------------------------------------
// Per-thread error message.
thread_local char g_last_error[512] = "";

qkn_status fail(qkn_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

qkn_status ok() {
    g_last_error[0] = '\0';
    return QKN_OK;
}

}  // namespace

namespace qkn {
// The calling thread's message for qknorm_last_error, for the library's other
// translation units (the host-buffer pipeline).
void set_last_error(const char *msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
}  // namespace qkn

namespace {

// Bytes of one element of x (and y), and of one element of gamma.
int elem_bytes(qkn_dtype dt) { return dt == QKN_F32 ? 4 : (dt == QKN_FP8_E4M3 ? 1 : 2); }
int gamma_bytes(qkn_dtype dt) { return dt == QKN_F32 ? 4 : 2; }

bool dtype_valid(int dt) { return dt >= QKN_F32 && dt <= QKN_FP8_E4M3; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


// ---------------------------------------------------------------------------
// Overlap of two row sets.
int64_t floor_div(int64_t a, int64_t b) {  // b > 0
    int64_t q = a / b;
    if ((a % b != 0) && (a < 0)) --q;
    return q;
}
int64_t ceil_div_signed(int64_t a, int64_t b) {  // b > 0
    return -floor_div(-a, b);
}

// Is there an integer k in [kmin, kmax] with lo < k * s < hi ?  (s > 0)
bool multiple_in_open_interval(int64_t s, int64_t lo, int64_t hi, int64_t kmin, int64_t kmax) {
    const int64_t k_lo = floor_div(lo, s) + 1;         // smallest k with k*s > lo
    const int64_t k_hi = ceil_div_signed(hi, s) - 1;   // largest k with k*s < hi
    const int64_t a = k_lo > kmin ? k_lo : kmin;
    const int64_t b = k_hi < kmax ? k_hi : kmax;
    return a <= b;
}

struct Region {
    uint64_t base;
    int64_t width;   // bytes per row
    int64_t stride;  // bytes between rows
    int64_t rows;
};

bool overlap(const Region &a, const Region &b) {
    if (a.rows < 1 || b.rows < 1 || a.width < 1 || b.width < 1) return false;
    const __int128 a_end = (__int128)a.base + (__int128)(a.rows - 1) * a.stride + a.width;
    const __int128 b_end = (__int128)b.base + (__int128)(b.rows - 1) * b.stride + b.width;
    if (a_end <= (__int128)b.base || b_end <= (__int128)a.base) return false;
    if (a.rows == 1 && b.rows == 1) return true;
    if (a.rows == 1 || b.rows == 1 || a.stride == b.stride) {
        // Rows of `m` (multi-row, stride s) against rows of `o`.  Row pair
        // (i, j) overlaps iff -w_m < (o + j*s_o) - (m + i*s) < w_o; with one
        // row in `o` (j = 0) or a shared stride this depends on one integer k.
        const Region &m = (a.rows == 1) ? b : a;
        const Region &o = (a.rows == 1) ? a : b;
        const int64_t s = m.stride;
        const int64_t d = (int64_t)(o.base - m.base);  // wraps correctly for nearby addresses
        int64_t kmin, kmax;
        if (o.rows == 1) {
            // i*s in (d - w_m, d + w_o), i in [0, rows_m - 1]
            kmin = 0;
            kmax = m.rows - 1;
            return multiple_in_open_interval(s, d - m.width, d + o.width, kmin, kmax);
        }
        // shared stride: (i - j)*s in (d - w_m, d + w_o), i - j in [-(rows_o-1), rows_m-1]
        kmin = -(o.rows - 1);
        kmax = m.rows - 1;
        return multiple_in_open_interval(s, d - m.width, d + o.width, kmin, kmax);
    }
    return true;  // different strides with intersecting ranges: conservative
}

// ---------------------------------------------------------------------------
// Device facts, cached per device.
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sm_count = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

struct OccEntry {
    const void *fn;
    int device;
    int threads;
    int64_t smem;
    int blocks;
};
constexpr int kOccSlots = 512;
OccEntry g_occ[kOccSlots];
int g_occ_n = 0;
std::mutex g_occ_mu;

qkn_status current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (*dev < 0 || *dev >= kMaxDevices) return fail(QKN_ERR_UNSUPPORTED, "device ordinal %d too large", *dev);
    return QKN_OK;
}

qkn_status sm_count(int dev, int *out) {
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (g_dev[dev].sm_count > 0) {
            *out = g_dev[dev].sm_count;
            return QKN_OK;
        }
    }
    int n = 0;
    cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess || n < 1)
        return fail(QKN_ERR_CUDA, "cudaDeviceGetAttribute(SM count): %s", cudaGetErrorString(e));
    std::lock_guard<std::mutex> lk(g_dev_mu);
    g_dev[dev].sm_count = n;
    *out = n;
    return QKN_OK;
}

qkn_status blocks_per_sm(const void *fn, int dev, int threads, int64_t dyn_smem, int *out) {
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        for (int i = 0; i < g_occ_n; ++i)
            if (g_occ[i].fn == fn && g_occ[i].device == dev && g_occ[i].threads == threads &&
                g_occ[i].smem == dyn_smem) {
                *out = g_occ[i].blocks;
                return QKN_OK;
            }
    }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, (size_t)dyn_smem);
    if (e != cudaSuccess)
        return fail(QKN_ERR_CUDA, "cudaOccupancyMaxActiveBlocksPerMultiprocessor: %s", cudaGetErrorString(e));
    if (n < 1) return fail(QKN_ERR_UNSUPPORTED, "kernel cannot run with %d threads per CTA", threads);
    std::lock_guard<std::mutex> lk(g_occ_mu);
    if (g_occ_n < kOccSlots) g_occ[g_occ_n++] = OccEntry{fn, dev, threads, dyn_smem, n};
    *out = n;
    return QKN_OK;
}

// ---------------------------------------------------------------------------
// Kernel selection.
template <typename E, int MODE, bool TAIL, int SETS>
const void *register_kernel(int nv) {
    switch (nv) {
        case 1: return (const void *)qkn::rows_register_kernel<E, 1, MODE, TAIL, SETS>;
        case 2: return (const void *)qkn::rows_register_kernel<E, 2, MODE, TAIL, SETS>;
        case 4: return (const void *)qkn::rows_register_kernel<E, 4, MODE, TAIL, SETS>;
        case 8: return (const void *)qkn::rows_register_kernel<E, 8, MODE, TAIL, SETS>;
        case 5:  // one warp per row of 129..160 vectors (a partial-sum or apply pass over shards)
            if constexpr (MODE == qkn::kFused) return nullptr;
            else return (const void *)qkn::rows_register_kernel<E, 5, MODE, TAIL, SETS>;
        default: return nullptr;
    }
}

// The two-pass kernels take one Q and one K row set only; multi-shard calls
// (SETS > 2) run the register kernel.
template <typename E, int MODE, int SETS>
const void *kernel_for(const qkn_launch &L, bool tail) {
    switch (L.kernel) {
        case QKN_KERNEL_REGISTER:
            return tail ? register_kernel<E, MODE, true, SETS>(L.vec_per_thread)
                        : register_kernel<E, MODE, false, SETS>(L.vec_per_thread);
        case QKN_KERNEL_TWOPASS_VEC:
            if constexpr (SETS == 2) return (const void *)qkn::rows_twopass_kernel<E, true, MODE>;
            return nullptr;
        case QKN_KERNEL_TWOPASS_SCALAR:
            if constexpr (SETS == 2) return (const void *)qkn::rows_twopass_kernel<E, false, MODE>;
            return nullptr;
        default: return nullptr;
    }
}

template <int MODE, int SETS = 2>
const void *kernel_for(qkn_dtype dt, const qkn_launch &L, bool tail) {
    switch (dt) {
        case QKN_F32: return kernel_for<float, MODE, SETS>(L, tail);
        case QKN_BF16: return kernel_for<__nv_bfloat16, MODE, SETS>(L, tail);
        case QKN_F16: return kernel_for<__half, MODE, SETS>(L, tail);
        case QKN_FP8_E4M3: return kernel_for<__nv_fp8_e4m3, MODE, SETS>(L, tail);
        default: return nullptr;
    }
}

// A prepared call: parameters plus the facts planning needs.
template <int SETS>
struct CallT {
    qkn::ParamsT<SETS> p;
    qkn_dtype dtype;
    bool vectorized;
    bool tail;          // some row ends in a partial 16-byte vector
    int64_t units_max;  // widest row in vectors (vectorized) or elements
};
using Call = CallT<2>;
using ShardCall = CallT<qkn::kMaxShardSets>;

// Zeroed call with `nsets` row sets in use.
template <int SETS>
void init_call(CallT<SETS> &c, qkn_dtype dtype, int nsets) {
    std::memset(&c, 0, sizeof(c));
    c.dtype = dtype;
    c.p.nsets = nsets;
}

void fill_rowset(qkn::RowSet &s, const void *in, void *out, const void *gamma, int64_t stride, int32_t width,
                 int32_t div_width, int esz) {
    const int per_vec = 16 / esz;
    s.in = static_cast<const char *>(in);
    s.out = static_cast<char *>(out);
    s.gamma = static_cast<const char *>(gamma);
    s.sumsq = nullptr;
    s.stride_bytes = stride * esz;
    s.width = width;
    s.nfull = width / per_vec;
    s.tail = width % per_vec;
    s.inv_div = static_cast<float>(1.0 / static_cast<double>(div_width));
    s.heads = 1;
    s.head_bytes = 0;
    s.rows = 0;
}

// Rows per set, and whether every set moves as 16-byte vectors (`aligned`:
// the caller's pointers and strides allow it), the widest row, any tail.
template <int SETS>
void finish_sets(CallT<SETS> &c, int esz, bool aligned) {
    bool v = aligned;
    int64_t w = 0;
    c.tail = false;
    for (int i = 0; i < c.p.nsets; ++i) {
        qkn::RowSet &d = c.p.set[i];
        d.rows = c.p.T * d.heads;
        if (d.heads > 1 && d.head_bytes % 16 != 0) v = false;  // every head must start on a vector
        if (d.width > w) w = d.width;
        if (d.tail) c.tail = true;
    }
    c.vectorized = v;
    const int per_vec = 16 / esz;
    c.units_max = v ? (w + per_vec - 1) / per_vec : w;
}

void finish_call(Call &c, int esz, std::initializer_list<const void *> ptrs, int64_t q_stride, int64_t k_stride) {
    bool v = ((q_stride * esz) % 16 == 0) && ((k_stride * esz) % 16 == 0);
    for (const void *p : ptrs)
        if (p && !aligned16(p)) v = false;
    finish_sets(c, esz, v);
}

// Row groups of the register kernel for a launch of `threads` threads with
// `nv` vectors each: the smallest group (a multiple of 32 dividing the CTA)
// whose threads cover the set's row, and the items that follow.
template <int SETS>
void set_groups(qkn::ParamsT<SETS> &p, int threads, int nv) {
    int64_t end = 0;
    for (int w = 0; w < p.nsets; ++w) {
        qkn::RowSet &d = p.set[w];
        const int64_t units = (int64_t)d.nfull + (d.tail ? 1 : 0);
        int group = threads;
        for (int g = 1; g < threads; g = g < 32 ? g * 2 : g + 32)
            if (threads % g == 0 && (int64_t)g * nv >= units) {
                group = g;
                break;
            }
        d.group = group;
        d.rows_per_item = threads / group;
        end += (d.rows + d.rows_per_item - 1) / d.rows_per_item;  // items: rows_per_item rows each
        d.item_end = end;
    }
    p.n_items = end;
}

bool eps_valid(float eps) { return std::isfinite(eps) && eps >= 0.0f; }

// Rows of T must stay addressable: (T - 1) * stride + width elements in bytes below 2^62.
bool extent_ok(int64_t T, int64_t stride, int64_t width, int esz) {
    if (T <= 0) return true;
    const __int128 bytes = ((__int128)(T - 1) * stride + width) * esz;
    return bytes < ((__int128)1 << 62);
}

Region rows_region(const void *base, int64_t width, int64_t stride, int64_t T, int esz) {
    return Region{(uint64_t)(uintptr_t)base, width * esz, stride * esz, T};
}
Region flat_region(const void *base, int64_t bytes) {
    return Region{(uint64_t)(uintptr_t)base, bytes, bytes, 1};
}

// Written region `w` against a region `r` it must not touch, unless `r` is
// the very same buffer (in place).
bool bad_overlap(const Region &w, const Region &r, bool allow_identical) {
    if (allow_identical && w.base == r.base && w.stride == r.stride && w.width == r.width) return false;
    return overlap(w, r);
}

// Common checks of the fused and apply forms: outputs vs everything else.
qkn_status check_outputs(const Region &oq, const Region &ok_, const Region &iq, const Region &ik,
                         const Region *others, int n_others) {
    if (overlap(oq, ok_)) return fail(QKN_ERR_INVALID_ARG, "q_out and k_out overlap");
    if (bad_overlap(oq, iq, true)) return fail(QKN_ERR_INVALID_ARG, "q_out partly overlaps q_in (only out == in is allowed)");
    if (bad_overlap(ok_, ik, true)) return fail(QKN_ERR_INVALID_ARG, "k_out partly overlaps k_in (only out == in is allowed)");
    if (overlap(oq, ik)) return fail(QKN_ERR_INVALID_ARG, "q_out overlaps k_in");
    if (overlap(ok_, iq)) return fail(QKN_ERR_INVALID_ARG, "k_out overlaps q_in");
    for (int i = 0; i < n_others; ++i) {
        if (overlap(oq, others[i])) return fail(QKN_ERR_INVALID_ARG, "q_out overlaps a read-only operand (gamma or sums)");
        if (overlap(ok_, others[i])) return fail(QKN_ERR_INVALID_ARG, "k_out overlaps a read-only operand (gamma or sums)");
    }
    return QKN_OK;
}

qkn_status prepare_layerwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                             const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                             int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype, Call &c) {
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (Hq <= 0 || Hk <= 0) return fail(QKN_ERR_INVALID_ARG, "widths must be positive (Hq = %d, Hk = %d)", Hq, Hk);
    if (q_stride < Hq || k_stride < Hk)
        return fail(QKN_ERR_INVALID_ARG, "row stride below width (q: %lld < %d or k: %lld < %d)",
                    (long long)q_stride, Hq, (long long)k_stride, Hk);
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, Hq, esz) || !extent_ok(T, k_stride, Hk, esz))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T > 0 && (!q_in || !q_out || !gamma_q || !k_in || !k_out || !gamma_k))
        return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (T > 0) {
        const Region iq = rows_region(q_in, Hq, q_stride, T, esz), oq = rows_region(q_out, Hq, q_stride, T, esz);
        const Region ik = rows_region(k_in, Hk, k_stride, T, esz), ok_ = rows_region(k_out, Hk, k_stride, T, esz);
        const int gsz = gamma_bytes(dtype);
        const Region others[2] = {flat_region(gamma_q, (int64_t)Hq * gsz), flat_region(gamma_k, (int64_t)Hk * gsz)};
        qkn_status st = check_outputs(oq, ok_, iq, ik, others, 2);
        if (st != QKN_OK) return st;
    }
    init_call(c, dtype, 2);
    fill_rowset(c.p.set[0], q_in, q_out, gamma_q, q_stride, Hq, Hq, esz);
    fill_rowset(c.p.set[1], k_in, k_out, gamma_k, k_stride, Hk, Hk, esz);
    c.p.T = T;
    c.p.eps = eps;
    c.p.set[0].P = 1;
    c.p.set[1].P = 1;
    finish_call(c, esz, {q_in, q_out, gamma_q, k_in, k_out, gamma_k}, q_stride, k_stride);
    return QKN_OK;
}

template <int MODE, int SETS>
qkn_status plan_call(const CallT<SETS> &c, qkn_launch &L) {
    int dev = 0, sms = 0, bps = 0;
    qkn_status st = current_device(&dev);
    if (st != QKN_OK) return st;
    if ((st = sm_count(dev, &sms)) != QKN_OK) return st;
    int64_t items = 0;
    for (int i = 0; i < c.p.nsets; ++i) items += c.p.set[i].rows;
    if ((st = qknorm_plan_shape(items, c.units_max, c.vectorized ? 1 : 0, sms, elem_bytes(c.dtype), &L)) !=
        QKN_OK)
        return fail(st, "planning failed");
    if (MODE == qkn::kStats && L.kernel == QKN_KERNEL_REGISTER && items > sms) {
        // The partial-sum pass only reads and holds no gamma: more vectors per
        // lane (up to 8; 4 for 1-byte elements) keep more bytes in flight,
        // one warp (or fewer lanes) per row, 128-thread CTAs.
        const int cap = elem_bytes(c.dtype) == 1 ? 4 : 8;
        int nv = 1;
        while (nv < cap && (int64_t)nv * 32 < c.units_max) nv *= 2;
        if ((int64_t)nv * 128 >= c.units_max) {
            L.vec_per_thread = nv;
            L.threads = 128;
        }
    }
    int oversubscribe = 1;  // CTAs per resident slot
    if (MODE == qkn::kApply && L.kernel == QKN_KERNEL_REGISTER && items > sms && c.units_max > 128 &&
        c.units_max <= 160) {
        // Rows of 129..160 vectors (a hidden dimension split into shards):
        // one warp per row with 5 vectors per lane covers it without idle
        // lanes or a CTA barrier; 8 rows per CTA, and four CTAs per resident
        // slot, so that CTAs finishing early take the next ones and the
        // ragged end of the row list spreads over the SMs.  (One B200, the
        // GQA step's apply pass over 4 + 4 shards of 1280 + 256 bf16 columns
        // for 16384 tokens: 62.8 us against 68.0 us for 2 vectors per lane in
        // 96-thread CTAs at one CTA per slot.)
        L.vec_per_thread = 5;
        L.threads = 256;
        oversubscribe = 4;
    }
    const void *fn = kernel_for<MODE, SETS>(c.dtype, L, c.tail);
    if (!fn) return fail(QKN_ERR_UNSUPPORTED, "no kernel for the planned launch");
    if ((st = blocks_per_sm(fn, dev, L.threads, 0, &bps)) != QKN_OK) return st;
    int64_t work = items;
    if (L.kernel == QKN_KERNEL_REGISTER) {  // narrow rows share CTAs: count items, not rows
        qkn::ParamsT<SETS> p = c.p;
        set_groups(p, L.threads, L.vec_per_thread);
        work = p.n_items;
    }
    if (MODE == qkn::kFused && L.kernel == QKN_KERNEL_REGISTER && work >= 4 * (int64_t)bps * sms) {
        // At least 4 items per resident slot: launch 3 (below 6 items per
        // slot) or 4 CTAs per slot rather than one persistent CTA, so the
        // hardware hands the remaining items to whichever CTAs finish first.
        // (One B200, graph replays, CTAs per slot 1 / 3 / 4: prefill T=4096
        // H=4096 bf16, 6.9 items per slot, 22.7-22.9 / 22.9 / 22.2-22.3 us;
        // packed T=4096, 4.3 items per slot, 15.5 / 14.7 / 15.0-15.1;
        // headwise T=4096, 4.3 items per slot, 15.1-15.2 / 14.6 / 14.9; with
        // fewer items per slot -- E4M3 prefill, packed T=1024 -- it did not
        // help.)
        oversubscribe = work < 6 * (int64_t)bps * sms ? 3 : 4;
    }
    L.grid = qknorm_plan_grid(work, bps * oversubscribe, sms);
    return QKN_OK;
}

template <int MODE, int SETS>
qkn_status check_launch(const CallT<SETS> &c, const qkn_launch &L) {
    if (L.threads < 32 || L.threads > 1024 || (L.threads % 32) != 0)
        return fail(QKN_ERR_INVALID_ARG, "threads must be a multiple of 32 in [32, 1024], got %d", L.threads);
    if (L.grid < 1 || L.grid > 2147483647LL) return fail(QKN_ERR_INVALID_ARG, "grid out of range");
    switch (L.kernel) {
        case QKN_KERNEL_REGISTER: {
            const int mt = qknorm_register_max_threads(L.vec_per_thread);
            if (mt == 0 || (MODE == qkn::kFused && L.vec_per_thread == 5))
                return fail(QKN_ERR_INVALID_ARG, MODE == qkn::kFused ? "vec_per_thread must be 1, 2, 4 or 8"
                                                                     : "vec_per_thread must be 1, 2, 4, 5 or 8");
            if (L.threads > mt) return fail(QKN_ERR_INVALID_ARG, "threads above %d for vec_per_thread %d", mt, L.vec_per_thread);
            if (!c.vectorized) return fail(QKN_ERR_INVALID_ARG, "register kernel needs 16-byte aligned buffers");
            if ((int64_t)L.vec_per_thread * L.threads < c.units_max)
                return fail(QKN_ERR_INVALID_ARG, "row of %lld vectors exceeds vec_per_thread * threads",
                            (long long)c.units_max);
            return QKN_OK;
        }
        case QKN_KERNEL_TWOPASS_VEC:
            if (!c.vectorized) return fail(QKN_ERR_INVALID_ARG, "vector kernel needs 16-byte aligned buffers");
            return QKN_OK;
        case QKN_KERNEL_TWOPASS_SCALAR: return QKN_OK;
        default: return fail(QKN_ERR_INVALID_ARG, "unknown kernel kind %d", L.kernel);
    }
}

// Every launch allows programmatic dependent launch: the kernel may be
// dispatched while the previous kernel in the stream drains (see
// pdl_wait_and_release in the kernels, which restores the ordering).
template <typename P>
cudaError_t launch_pdl(const void *fn, unsigned grid, unsigned block, size_t smem, cudaStream_t s, const P &p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {const_cast<P *>(&p)};
    return cudaLaunchKernelExC(&cfg, fn, args);
}

template <int MODE, int SETS>
cudaError_t launch_any(const qkn_launch &L, const CallT<SETS> &c, cudaStream_t s) {
    const void *fn = kernel_for<MODE, SETS>(c.dtype, L, c.tail);
    if (!fn) return cudaErrorInvalidValue;
    qkn::ParamsT<SETS> p = c.p;
    if (L.kernel == QKN_KERNEL_REGISTER) set_groups(p, L.threads, L.vec_per_thread);
    return launch_pdl(fn, (unsigned)L.grid, (unsigned)L.threads, 0, s, p);
}

template <int MODE, int SETS>
qkn_status launch(const CallT<SETS> &c, const qkn_launch &L, void *stream) {
    cudaError_t e = launch_any<MODE, SETS>(L, c, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

qkn_status prepare_stats(const void *q_shard, int64_t q_stride, int32_t hq_shard, float *q_sumsq,
                         const void *k_shard, int64_t k_stride, int32_t hk_shard, float *k_sumsq, int64_t T,
                         qkn_dtype dtype, Call &c) {
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (hq_shard <= 0 || hk_shard <= 0) return fail(QKN_ERR_INVALID_ARG, "shard widths must be positive");
    if (q_stride < hq_shard || k_stride < hk_shard) return fail(QKN_ERR_INVALID_ARG, "row stride below shard width");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, hq_shard, esz) || !extent_ok(T, k_stride, hk_shard, esz))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T > 0 && (!q_shard || !q_sumsq || !k_shard || !k_sumsq)) return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (T > 0) {
        const Region iq = rows_region(q_shard, hq_shard, q_stride, T, esz);
        const Region ik = rows_region(k_shard, hk_shard, k_stride, T, esz);
        const Region sq = flat_region(q_sumsq, T * 4), sk = flat_region(k_sumsq, T * 4);
        if (overlap(sq, sk)) return fail(QKN_ERR_INVALID_ARG, "q_sumsq and k_sumsq overlap");
        if (overlap(sq, iq) || overlap(sq, ik) || overlap(sk, iq) || overlap(sk, ik))
            return fail(QKN_ERR_INVALID_ARG, "a sum array overlaps an input");
    }
    init_call(c, dtype, 2);
    fill_rowset(c.p.set[0], q_shard, nullptr, nullptr, q_stride, hq_shard, hq_shard, esz);
    fill_rowset(c.p.set[1], k_shard, nullptr, nullptr, k_stride, hk_shard, hk_shard, esz);
    c.p.set[0].sumsq = q_sumsq;
    c.p.set[1].sumsq = k_sumsq;
    c.p.T = T;
    c.p.eps = 0.0f;
    c.p.set[0].P = 1;
    c.p.set[1].P = 1;
    finish_call(c, esz, {q_shard, k_shard}, q_stride, k_stride);
    return QKN_OK;
}

qkn_status prepare_apply(const void *q_in, void *q_out, const void *gamma_q_shard, int64_t q_stride,
                         int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full, const void *k_in, void *k_out,
                         const void *gamma_k_shard, int64_t k_stride, int32_t hk_shard, const float *k_sumsq_all,
                         int32_t Hk_full, int32_t P, int64_t T, float eps, qkn_dtype dtype, Call &c) {
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (P < 1) return fail(QKN_ERR_INVALID_ARG, "P = %d < 1", P);
    if (hq_shard <= 0 || hk_shard <= 0) return fail(QKN_ERR_INVALID_ARG, "shard widths must be positive");
    if (Hq_full < hq_shard || Hk_full < hk_shard) return fail(QKN_ERR_INVALID_ARG, "full width below shard width");
    if (q_stride < hq_shard || k_stride < hk_shard) return fail(QKN_ERR_INVALID_ARG, "row stride below shard width");
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, hq_shard, esz) || !extent_ok(T, k_stride, hk_shard, esz) ||
        !extent_ok(1, 0, (int64_t)P * T, 4))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T > 0 && (!q_in || !q_out || !gamma_q_shard || !q_sumsq_all || !k_in || !k_out || !gamma_k_shard ||
                  !k_sumsq_all))
        return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (T > 0) {
        const Region iq = rows_region(q_in, hq_shard, q_stride, T, esz);
        const Region oq = rows_region(q_out, hq_shard, q_stride, T, esz);
        const Region ik = rows_region(k_in, hk_shard, k_stride, T, esz);
        const Region ok_ = rows_region(k_out, hk_shard, k_stride, T, esz);
        const int gsz = gamma_bytes(dtype);
        const Region others[4] = {flat_region(gamma_q_shard, (int64_t)hq_shard * gsz),
                                  flat_region(gamma_k_shard, (int64_t)hk_shard * gsz),
                                  flat_region(q_sumsq_all, (int64_t)P * T * 4),
                                  flat_region(k_sumsq_all, (int64_t)P * T * 4)};
        qkn_status st = check_outputs(oq, ok_, iq, ik, others, 4);
        if (st != QKN_OK) return st;
    }
    init_call(c, dtype, 2);
    fill_rowset(c.p.set[0], q_in, q_out, gamma_q_shard, q_stride, hq_shard, Hq_full, esz);
    fill_rowset(c.p.set[1], k_in, k_out, gamma_k_shard, k_stride, hk_shard, Hk_full, esz);
    c.p.set[0].sumsq_all = q_sumsq_all;
    c.p.set[1].sumsq_all = k_sumsq_all;
    c.p.T = T;
    c.p.eps = eps;
    c.p.set[0].P = P;
    c.p.set[1].P = P;
    finish_call(c, esz, {q_in, q_out, gamma_q_shard, k_in, k_out, gamma_k_shard}, q_stride, k_stride);
    return QKN_OK;
}

// Multi-shard forms: P shards of Q and P of K, each shard's rows in its own
// buffer (same width and stride for every shard of a tensor), in one launch.
qkn_status check_shard_common(int32_t P, int64_t T, int32_t hq_shard, int32_t hk_shard, int64_t q_stride,
                              int64_t k_stride, qkn_dtype dtype) {
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (P < 1 || P > qkn::kMaxShards) return fail(QKN_ERR_INVALID_ARG, "P = %d outside [1, %d]", P, qkn::kMaxShards);
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (hq_shard <= 0 || hk_shard <= 0) return fail(QKN_ERR_INVALID_ARG, "shard widths must be positive");
    if (q_stride < hq_shard || k_stride < hk_shard) return fail(QKN_ERR_INVALID_ARG, "row stride below shard width");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, hq_shard, esz) || !extent_ok(T, k_stride, hk_shard, esz) ||
        !extent_ok(1, 0, (int64_t)P * T, 4))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    return QKN_OK;
}

bool shard_ptrs_aligned(const void *const *a, int P) {
    for (int p = 0; p < P; ++p)
        if (!aligned16(a[p])) return false;
    return true;
}

qkn_status prepare_stats_shards(int32_t P, const void *const *q_shards, int64_t q_stride, int32_t hq_shard,
                                float *q_sumsq_all, const void *const *k_shards, int64_t k_stride, int32_t hk_shard,
                                float *k_sumsq_all, int64_t T, qkn_dtype dtype, ShardCall &c) {
    qkn_status st = check_shard_common(P, T, hq_shard, hk_shard, q_stride, k_stride, dtype);
    if (st != QKN_OK) return st;
    const int esz = elem_bytes(dtype);
    if (T > 0) {
        if (!q_shards || !k_shards || !q_sumsq_all || !k_sumsq_all) return fail(QKN_ERR_INVALID_ARG, "null pointer");
        for (int p = 0; p < P; ++p)
            if (!q_shards[p] || !k_shards[p]) return fail(QKN_ERR_INVALID_ARG, "null shard pointer %d", p);
        const Region sq = flat_region(q_sumsq_all, (int64_t)P * T * 4), sk = flat_region(k_sumsq_all, (int64_t)P * T * 4);
        if (overlap(sq, sk)) return fail(QKN_ERR_INVALID_ARG, "q_sumsq_all and k_sumsq_all overlap");
        for (int p = 0; p < P; ++p) {
            const Region iq = rows_region(q_shards[p], hq_shard, q_stride, T, esz);
            const Region ik = rows_region(k_shards[p], hk_shard, k_stride, T, esz);
            if (overlap(sq, iq) || overlap(sq, ik) || overlap(sk, iq) || overlap(sk, ik))
                return fail(QKN_ERR_INVALID_ARG, "a sum array overlaps shard %d", p);
        }
    }
    init_call(c, dtype, 2 * P);
    for (int p = 0; p < P && T > 0; ++p) {
        qkn::RowSet &dq = c.p.set[p], &dk = c.p.set[P + p];
        fill_rowset(dq, q_shards[p], nullptr, nullptr, q_stride, hq_shard, hq_shard, esz);
        fill_rowset(dk, k_shards[p], nullptr, nullptr, k_stride, hk_shard, hk_shard, esz);
        dq.sumsq = q_sumsq_all + (int64_t)p * T;
        dk.sumsq = k_sumsq_all + (int64_t)p * T;
        dq.P = dk.P = 1;
    }
    c.p.T = T;
    c.p.eps = 0.0f;
    if (T > 0)
        finish_sets(c, esz, (q_stride * esz) % 16 == 0 && (k_stride * esz) % 16 == 0 &&
                                shard_ptrs_aligned(q_shards, P) && shard_ptrs_aligned(k_shards, P));
    return QKN_OK;
}

qkn_status prepare_apply_shards(int32_t P, const void *const *q_in, void *const *q_out,
                                const void *const *gamma_q_shards, int64_t q_stride, int32_t hq_shard,
                                const float *q_sumsq_all, int32_t Hq_full, const void *const *k_in,
                                void *const *k_out, const void *const *gamma_k_shards, int64_t k_stride,
                                int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full, int64_t T, float eps,
                                qkn_dtype dtype, ShardCall &c) {
    qkn_status st = check_shard_common(P, T, hq_shard, hk_shard, q_stride, k_stride, dtype);
    if (st != QKN_OK) return st;
    if (Hq_full < hq_shard || Hk_full < hk_shard) return fail(QKN_ERR_INVALID_ARG, "full width below shard width");
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const int esz = elem_bytes(dtype);
    const int gsz = gamma_bytes(dtype);
    if (T > 0) {
        if (!q_in || !q_out || !gamma_q_shards || !k_in || !k_out || !gamma_k_shards || !q_sumsq_all || !k_sumsq_all)
            return fail(QKN_ERR_INVALID_ARG, "null pointer");
        for (int p = 0; p < P; ++p)
            if (!q_in[p] || !q_out[p] || !gamma_q_shards[p] || !k_in[p] || !k_out[p] || !gamma_k_shards[p])
                return fail(QKN_ERR_INVALID_ARG, "null pointer for shard %d", p);
        // every output against everything else of every shard (its own input
        // only when identical: in place)
        for (int p = 0; p < P; ++p) {
            const Region oq = rows_region(q_out[p], hq_shard, q_stride, T, esz);
            const Region ok_ = rows_region(k_out[p], hk_shard, k_stride, T, esz);
            for (int o = 0; o < P; ++o) {
                const Region iq = rows_region(q_in[o], hq_shard, q_stride, T, esz);
                const Region ik = rows_region(k_in[o], hk_shard, k_stride, T, esz);
                const Region others[4] = {flat_region(gamma_q_shards[o], (int64_t)hq_shard * gsz),
                                          flat_region(gamma_k_shards[o], (int64_t)hk_shard * gsz),
                                          flat_region(q_sumsq_all, (int64_t)P * T * 4),
                                          flat_region(k_sumsq_all, (int64_t)P * T * 4)};
                if (o == p) {
                    if ((st = check_outputs(oq, ok_, iq, ik, others, 4)) != QKN_OK) return st;
                    continue;
                }
                const Region oq2 = rows_region(q_out[o], hq_shard, q_stride, T, esz);
                const Region ok2 = rows_region(k_out[o], hk_shard, k_stride, T, esz);
                const Region all[8] = {iq, ik, oq2, ok2, others[0], others[1], others[2], others[3]};
                for (const Region &r : all)
                    if (overlap(oq, r) || overlap(ok_, r))
                        return fail(QKN_ERR_INVALID_ARG, "an output of shard %d overlaps an operand of shard %d", p, o);
            }
        }
    }
    init_call(c, dtype, 2 * P);
    for (int p = 0; p < P && T > 0; ++p) {
        qkn::RowSet &dq = c.p.set[p], &dk = c.p.set[P + p];
        fill_rowset(dq, q_in[p], q_out[p], gamma_q_shards[p], q_stride, hq_shard, Hq_full, esz);
        fill_rowset(dk, k_in[p], k_out[p], gamma_k_shards[p], k_stride, hk_shard, Hk_full, esz);
        dq.sumsq_all = q_sumsq_all;
        dk.sumsq_all = k_sumsq_all;
        dq.P = dk.P = P;
    }
    c.p.T = T;
    c.p.eps = eps;
    if (T > 0) {
        bool v = (q_stride * esz) % 16 == 0 && (k_stride * esz) % 16 == 0;
        for (const void *const *a : {q_in, (const void *const *)q_out, gamma_q_shards, k_in,
                                     (const void *const *)k_out, gamma_k_shards})
            v = v && shard_ptrs_aligned(a, P);
        finish_sets(c, esz, v);
    }
    return QKN_OK;
}

// A multi-shard call runs as one launch of the register kernel when its rows
// allow it (16-byte aligned, at most 32 KB); otherwise shard by shard.
bool one_launch(const ShardCall &c) { return c.vectorized && c.units_max <= 2048; }

qkn_status prepare_headwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride, int32_t q_heads,
                            const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride, int32_t k_heads,
                            int64_t T, int32_t head_dim, float eps, qkn_dtype dtype, Call &c) {
    if (q_heads <= 0 || k_heads <= 0 || head_dim <= 0)
        return fail(QKN_ERR_INVALID_ARG, "heads and head_dim must be positive");
    const int64_t wq = (int64_t)q_heads * head_dim, wk = (int64_t)k_heads * head_dim;
    if (wq > INT32_MAX || wk > INT32_MAX) return fail(QKN_ERR_INVALID_ARG, "row width overflows");
    if (T > 0 && ((int64_t)T * q_heads >= ((int64_t)1 << 31) || (int64_t)T * k_heads >= ((int64_t)1 << 31)))
        return fail(QKN_ERR_INVALID_ARG, "T * heads must stay below 2^31");
    // Validate the whole rows as the layerwise form does (sizes, strides, overlaps),
    // with gamma regions of head_dim elements.
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (q_stride < wq || k_stride < wk) return fail(QKN_ERR_INVALID_ARG, "row stride below heads * head_dim");
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, wq, esz) || !extent_ok(T, k_stride, wk, esz))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T > 0 && (!q_in || !q_out || !gamma_q || !k_in || !k_out || !gamma_k))
        return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (T > 0) {
        const Region iq = rows_region(q_in, wq, q_stride, T, esz), oq = rows_region(q_out, wq, q_stride, T, esz);
        const Region ik = rows_region(k_in, wk, k_stride, T, esz), ok_ = rows_region(k_out, wk, k_stride, T, esz);
        const int gsz = gamma_bytes(dtype);
        const Region others[2] = {flat_region(gamma_q, (int64_t)head_dim * gsz),
                                  flat_region(gamma_k, (int64_t)head_dim * gsz)};
        qkn_status st = check_outputs(oq, ok_, iq, ik, others, 2);
        if (st != QKN_OK) return st;
    }
    init_call(c, dtype, 2);
    fill_rowset(c.p.set[0], q_in, q_out, gamma_q, q_stride, head_dim, head_dim, esz);
    fill_rowset(c.p.set[1], k_in, k_out, gamma_k, k_stride, head_dim, head_dim, esz);
    c.p.set[0].heads = q_heads;
    c.p.set[1].heads = k_heads;
    c.p.set[0].head_bytes = (int64_t)head_dim * esz;
    c.p.set[1].head_bytes = (int64_t)head_dim * esz;
    c.p.T = T;
    c.p.eps = eps;
    c.p.set[0].P = 1;
    c.p.set[1].P = 1;
    finish_call(c, esz, {q_in, q_out, gamma_q, k_in, k_out, gamma_k}, q_stride, k_stride);
    return QKN_OK;
}

// ---------------------------------------------------------------------------
// QKV projection with Phase A sums in the epilogue.
constexpr int kTileN = qkn::gemm::kBN;
constexpr uint64_t kGemmTimeoutNs = 2000000000ull;  // 2 s per mbarrier wait

struct Projection {
    const void *x, *w;
    void *qkv;
    int64_t x_stride, w_stride, qkv_stride, T;
    int32_t D, Hq, Hk, Hv, N;
};

qkn_status prepare_projection(const void *x, int64_t x_stride, const void *w, int64_t w_stride, void *qkv,
                              int64_t qkv_stride, int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv,
                              qkn_dtype dtype, Projection &pr) {
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (dtype != QKN_BF16) return fail(QKN_ERR_UNSUPPORTED, "the projection runs on bfloat16 operands only");
    if (T < 0) return fail(QKN_ERR_INVALID_ARG, "T = %lld < 0", (long long)T);
    if (T >= ((int64_t)1 << 31)) return fail(QKN_ERR_INVALID_ARG, "T must stay below 2^31");
    if (D <= 0 || Hq <= 0 || Hk <= 0 || Hv < 0) return fail(QKN_ERR_INVALID_ARG, "D, Hq, Hk must be positive, Hv >= 0");
    if (Hq % kTileN || Hk % kTileN || Hv % kTileN)
        return fail(QKN_ERR_UNSUPPORTED, "Hq, Hk and Hv must be multiples of %d (the output tile)", kTileN);
    const int64_t N = (int64_t)Hq + Hk + Hv;
    if (N > INT32_MAX) return fail(QKN_ERR_INVALID_ARG, "Hq + Hk + Hv overflows");
    if (x_stride < D || w_stride < D || qkv_stride < N) return fail(QKN_ERR_INVALID_ARG, "row stride below width");
    if (((T + 127) / 128) * (N / kTileN) > ((int64_t)1 << 30))
        return fail(QKN_ERR_UNSUPPORTED, "more than 2^30 output tiles");
    if (!extent_ok(T, x_stride, D, 2) || !extent_ok(N, w_stride, D, 2) || !extent_ok(T, qkv_stride, N, 2))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T > 0 && (!x || !w || !qkv)) return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (T > 0 && (!aligned16(x) || !aligned16(w) || !aligned16(qkv) || (x_stride % 8) || (w_stride % 8) ||
                  (qkv_stride % 8)))
        return fail(QKN_ERR_INVALID_ARG, "x, w and qkv must be 16-byte aligned with strides a multiple of 8 elements");
    pr = Projection{x, w, qkv, x_stride, w_stride, qkv_stride, T, D, Hq, Hk, Hv, (int32_t)N};
    return QKN_OK;
}

// Regions the projection's outputs must not touch.
qkn_status check_projection_overlaps(const Projection &pr, const float *q_sums, const float *k_sums,
                                     const void *gamma_q, const void *gamma_k) {
    const Region rx = rows_region(pr.x, pr.D, pr.x_stride, pr.T, 2);
    const Region rw = rows_region(pr.w, pr.D, pr.w_stride, pr.N, 2);
    const Region ro = rows_region(pr.qkv, pr.N, pr.qkv_stride, pr.T, 2);
    const Region sq = flat_region(q_sums, (int64_t)(pr.Hq / kTileN) * pr.T * 4);
    const Region sk = flat_region(k_sums, (int64_t)(pr.Hk / kTileN) * pr.T * 4);
    if (overlap(ro, rx) || overlap(ro, rw)) return fail(QKN_ERR_INVALID_ARG, "qkv overlaps x or w");
    if (overlap(ro, sq) || overlap(ro, sk)) return fail(QKN_ERR_INVALID_ARG, "qkv overlaps the partial sums");
    if (overlap(sq, sk)) return fail(QKN_ERR_INVALID_ARG, "the Q and K partial sums overlap");
    if (overlap(sq, rx) || overlap(sq, rw) || overlap(sk, rx) || overlap(sk, rw))
        return fail(QKN_ERR_INVALID_ARG, "the partial sums overlap x or w");
    if (gamma_q || gamma_k) {
        const Region gq = flat_region(gamma_q, (int64_t)pr.Hq * 2), gk = flat_region(gamma_k, (int64_t)pr.Hk * 2);
        if (overlap(ro, gq) || overlap(ro, gk)) return fail(QKN_ERR_INVALID_ARG, "qkv overlaps gamma");
        if (overlap(sq, gq) || overlap(sq, gk) || overlap(sk, gq) || overlap(sk, gk))
            return fail(QKN_ERR_INVALID_ARG, "the partial sums overlap gamma");
    }
    return QKN_OK;
}

// The tile counts of a projection of T tokens, D inputs and Hq + Hk + Hv
// outputs (Hq, Hk, Hv multiples of kTileN).
void gemm_tiles(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, qkn::gemm::GemmParams &gp) {
    gp.T = T;
    gp.k_blocks = (D + qkn::gemm::kBK - 1) / qkn::gemm::kBK;
    gp.q_tiles = Hq / kTileN;
    gp.k_tiles = Hk / kTileN;
    gp.n_tiles = (Hq + Hk + Hv) / kTileN;
    gp.m_tiles = (int32_t)((T + qkn::gemm::kBM - 1) / qkn::gemm::kBM);
    gp.m_units = (int32_t)((T + qkn::gemm::kBM * qkn::gemm::kCta - 1) / (qkn::gemm::kBM * qkn::gemm::kCta));
    gp.num_units = gp.m_units * gp.n_tiles;
}

qkn_status check_gemm_shape(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv) {
    if (T < 1 || T >= ((int64_t)1 << 31)) return fail(QKN_ERR_INVALID_ARG, "T must be in [1, 2^31)");
    if (D <= 0 || Hq <= 0 || Hk <= 0 || Hv < 0) return fail(QKN_ERR_INVALID_ARG, "D, Hq, Hk must be positive, Hv >= 0");
    if (Hq % kTileN || Hk % kTileN || Hv % kTileN)
        return fail(QKN_ERR_UNSUPPORTED, "Hq, Hk and Hv must be multiples of %d (the output tile)", kTileN);
    const int64_t N = (int64_t)Hq + Hk + Hv;
    if (N > INT32_MAX) return fail(QKN_ERR_INVALID_ARG, "Hq + Hk + Hv overflows");
    if (((T + 127) / 128) * (N / kTileN) > ((int64_t)1 << 30))
        return fail(QKN_ERR_UNSUPPORTED, "more than 2^30 output tiles");
    return QKN_OK;
}

void fill_schedule(const qkn::gemm::GemmParams &gp, int32_t clusters, qkn_gemm_schedule *out) {
    out->clusters = gp.num_units < clusters ? gp.num_units : clusters;
    out->units = gp.num_units;
    out->group_units = gp.group_units;
}

qkn_status launch_projection_gemm(const Projection &pr, float *q_sums, float *k_sums, void *stream) {
    qkn::gemm::GemmParams gp{};
    gp.qkv = static_cast<char *>(pr.qkv);
    gp.qkv_stride_bytes = pr.qkv_stride * 2;
    gp.q_sumsq = q_sums;
    gp.k_sumsq = k_sums;
    gemm_tiles(pr.T, pr.D, pr.Hq, pr.Hk, pr.Hv, gp);
    gp.timeout_ns = kGemmTimeoutNs;
    const char *what = "";
    cudaError_t e = qkn::gemm::launch_qkv_gemm(pr.x, pr.x_stride, pr.w, pr.w_stride, pr.D, pr.N, gp,
                                               static_cast<cudaStream_t>(stream), &what);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "projection GEMM (%s): %s", what, cudaGetErrorString(e));
    return ok();
}

}  // namespace

// ===========================================================================
// ---------------------------------------------------------------------------
// Scratch for qknorm_qkv_projection_noalloc: a fixed array in the library's
// own device image, so that entry point never allocates.  Each GPU that loads
// the library holds it until the process exits.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in for the symbol);
// the device address comes from cudaGetSymbolAddress, looked up once per
// device and context.
constexpr int64_t kNoAllocScratchBytes = (int64_t)4 << 20;  // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / 4];

namespace {
constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;

struct ScratchAddr {
    unsigned long long ctx_id;  // the context the address belongs to (0: unknown)
    void *addr;
};
ScratchAddr g_scratch_addr[kMaxScratchDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// The unique id of the calling thread's current CUDA context, or 0 when there
// is none yet or the driver cannot tell.  A device reset (cudaDeviceReset)
// ends the primary context, and the next one gets a new id -- and a new
// address for the scratch array.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_noalloc_scratch on the current device: looked up with
// that device current on the first call, and again whenever the current
// context is not the one the cached address came from (after a device reset),
// or on every call when the context's id cannot be read.
qkn_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxScratchDevices) return fail(QKN_ERR_UNSUPPORTED, "device index %d too large", dev);
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ScratchAddr &slot = g_scratch_addr[dev];
    if (!slot.addr || ctx == 0 || slot.ctx_id != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(QKN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        // the lookup makes the device's primary context current if none was
        slot = ScratchAddr{ctx ? ctx : current_context_id(), p};
    }
    *out = slot.addr;
    return QKN_OK;
}
}  // namespace

extern "C" {

int32_t qknorm_register_max_threads(int32_t vec_per_thread) {
    switch (vec_per_thread) {
        case 1: return qkn::RegisterBounds<1>::kMaxThreads;
        case 2: return qkn::RegisterBounds<2>::kMaxThreads;
        case 4: return qkn::RegisterBounds<4>::kMaxThreads;
        case 8: return qkn::RegisterBounds<8>::kMaxThreads;
        case 5: return qkn::RegisterBounds<5>::kMaxThreads;
        default: return 0;
    }
}

qkn_status qknorm_plan_shape(int64_t rows, int64_t units_max, int32_t vectorized, int32_t sm_count,
                             int32_t elem_bytes, qkn_launch *out) {
    if (!out || rows < 1 || units_max < 1 || sm_count < 1) return QKN_ERR_INVALID_ARG;
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4) return QKN_ERR_INVALID_ARG;
    qkn_launch L{};
    L.grid = 0;
    auto round32 = [](int64_t n) { return (int32_t)(((n + 31) / 32) * 32); };
    if (!vectorized) {
        L.kernel = QKN_KERNEL_TWOPASS_SCALAR;
        L.vec_per_thread = 0;
        L.threads = units_max >= 256 ? 256 : round32(units_max);
        *out = L;
        return QKN_OK;
    }
    if (units_max > 2048) {  // beyond 32 KB per row: two passes
        L.kernel = QKN_KERNEL_TWOPASS_VEC;
        L.vec_per_thread = 0;
        L.threads = 512;
        *out = L;
        return QKN_OK;
    }
    L.kernel = QKN_KERNEL_REGISTER;
    int nv;
    bool narrow = false, many = false;
    if (rows <= sm_count) {
        // Few rows (decode): spread each row over many threads so a row costs
        // about one memory round trip (two vectors per thread measured best).
        nv = units_max < 128 ? 1 : 2;
    } else if (units_max < 64) {
        // Many narrow rows (attention heads, thin shards): a few lanes per row
        // with up to four vectors each, so every thread keeps 64 bytes in
        // flight, and several rows per warp.
        narrow = true;
        nv = 1;
        while (nv < 4 && nv < units_max) nv *= 2;
    } else {
        // Many rows: moderate CTAs, several vectors in flight per thread.
        nv = units_max >= 256 ? 4 : 2;
        many = true;
    }
    // A 16-byte vector of 1-byte elements widens to twice the fp32 registers:
    // hold half as many per thread -- except for many wide rows, whose gamma
    // is re-read per row instead of held (1-byte elements), which leaves room
    // for the full count and halves the per-row work per vector.
    if (elem_bytes == 1 && nv > 1 && !many) nv /= 2;
    int32_t threads = round32((units_max + nv - 1) / nv);
    while (threads > qknorm_register_max_threads(nv)) {
        nv *= 2;
        threads = round32((units_max + nv - 1) / nv);
    }
    if (narrow) threads = 256;  // a CTA holds many row groups
    L.vec_per_thread = nv;
    L.threads = threads;
    *out = L;
    return QKN_OK;
}

int64_t qknorm_plan_grid(int64_t rows, int32_t blocks_per_sm, int32_t sm_count) {
    if (rows < 1) return 0;
    const int64_t bps = blocks_per_sm > 0 ? blocks_per_sm : 1;
    const int64_t sms = sm_count > 0 ? sm_count : 1;
    const int64_t resident = bps * sms;
    return rows < resident ? rows : resident;
}

int qknorm_regions_overlap(uint64_t a_base, int64_t a_width, int64_t a_stride, int64_t a_rows,
                           uint64_t b_base, int64_t b_width, int64_t b_stride, int64_t b_rows) {
    Region a{a_base, a_width, a_stride, a_rows}, b{b_base, b_width, b_stride, b_rows};
    if (a.rows > 1 && a.stride < 1) return 1;
    if (b.rows > 1 && b.stride < 1) return 1;
    return overlap(a, b) ? 1 : 0;
}

qkn_status qknorm_layerwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                            const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                            int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype, void *stream) {
    Call c;
    qkn_status st = prepare_layerwise(q_in, q_out, gamma_q, q_stride, k_in, k_out, gamma_k, k_stride, T, Hq,
                                      Hk, eps, dtype, c);
    if (st != QKN_OK) return st;
    if (T == 0) return ok();
    qkn_launch L;
    if ((st = plan_call<qkn::kFused>(c, L)) != QKN_OK) return st;
    return launch<qkn::kFused>(c, L, stream);
}

qkn_status qknorm_layerwise_plan(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                 const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                 int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype,
                                 qkn_launch *out) {
    if (!out) return fail(QKN_ERR_INVALID_ARG, "null output");
    Call c;
    qkn_status st = prepare_layerwise(q_in, q_out, gamma_q, q_stride, k_in, k_out, gamma_k, k_stride, T, Hq,
                                      Hk, eps, dtype, c);
    if (st != QKN_OK) return st;
    if (T == 0) {
        std::memset(out, 0, sizeof(*out));
        return ok();
    }
    if ((st = plan_call<qkn::kFused>(c, *out)) != QKN_OK) return st;
    return ok();
}

qkn_status qknorm_layerwise_launch(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                   const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                   int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype, void *stream,
                                   const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    Call c;
    qkn_status st = prepare_layerwise(q_in, q_out, gamma_q, q_stride, k_in, k_out, gamma_k, k_stride, T, Hq,
                                      Hk, eps, dtype, c);
    if (st != QKN_OK) return st;
    if ((st = check_launch<qkn::kFused>(c, *launch_cfg)) != QKN_OK) return st;
    if (T == 0) return ok();
    return launch<qkn::kFused>(c, *launch_cfg, stream);
}

qkn_status qknorm_headwise(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride, int32_t q_heads,
                           const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride, int32_t k_heads,
                           int64_t T, int32_t head_dim, float eps, qkn_dtype dtype, void *stream) {
    Call c;
    qkn_status st = prepare_headwise(q_in, q_out, gamma_q, q_stride, q_heads, k_in, k_out, gamma_k, k_stride,
                                     k_heads, T, head_dim, eps, dtype, c);
    if (st != QKN_OK) return st;
    if (T == 0) return ok();
    qkn_launch L;
    if ((st = plan_call<qkn::kFused>(c, L)) != QKN_OK) return st;
    return launch<qkn::kFused>(c, L, stream);
}

qkn_status qknorm_headwise_launch(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                  int32_t q_heads, const void *k_in, void *k_out, const void *gamma_k,
                                  int64_t k_stride, int32_t k_heads, int64_t T, int32_t head_dim, float eps,
                                  qkn_dtype dtype, void *stream, const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    Call c;
    qkn_status st = prepare_headwise(q_in, q_out, gamma_q, q_stride, q_heads, k_in, k_out, gamma_k, k_stride,
                                     k_heads, T, head_dim, eps, dtype, c);
    if (st != QKN_OK) return st;
    if ((st = check_launch<qkn::kFused>(c, *launch_cfg)) != QKN_OK) return st;
    if (T == 0) return ok();
    return launch<qkn::kFused>(c, *launch_cfg, stream);
}

qkn_status qknorm_partial_stats(const void *q_shard, int64_t q_stride, int32_t hq_shard, float *q_sumsq,
                                const void *k_shard, int64_t k_stride, int32_t hk_shard, float *k_sumsq,
                                int64_t T, qkn_dtype dtype, void *stream) {
    Call c;
    qkn_status st = prepare_stats(q_shard, q_stride, hq_shard, q_sumsq, k_shard, k_stride, hk_shard, k_sumsq, T,
                                  dtype, c);
    if (st != QKN_OK) return st;
    if (T == 0) return ok();
    qkn_launch L;
    if ((st = plan_call<qkn::kStats>(c, L)) != QKN_OK) return st;
    return launch<qkn::kStats>(c, L, stream);
}

qkn_status qknorm_partial_stats_launch(const void *q_shard, int64_t q_stride, int32_t hq_shard, float *q_sumsq,
                                       const void *k_shard, int64_t k_stride, int32_t hk_shard, float *k_sumsq,
                                       int64_t T, qkn_dtype dtype, void *stream, const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    Call c;
    qkn_status st = prepare_stats(q_shard, q_stride, hq_shard, q_sumsq, k_shard, k_stride, hk_shard, k_sumsq, T,
                                  dtype, c);
    if (st != QKN_OK) return st;
    if ((st = check_launch<qkn::kStats>(c, *launch_cfg)) != QKN_OK) return st;
    if (T == 0) return ok();
    return launch<qkn::kStats>(c, *launch_cfg, stream);
}

qkn_status qknorm_combine_apply(const void *q_in, void *q_out, const void *gamma_q_shard, int64_t q_stride,
                                int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full,
                                const void *k_in, void *k_out, const void *gamma_k_shard, int64_t k_stride,
                                int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full,
                                int32_t P, int64_t T, float eps, qkn_dtype dtype, void *stream) {
    Call c;
    qkn_status st = prepare_apply(q_in, q_out, gamma_q_shard, q_stride, hq_shard, q_sumsq_all, Hq_full, k_in, k_out,
                                  gamma_k_shard, k_stride, hk_shard, k_sumsq_all, Hk_full, P, T, eps, dtype, c);
    if (st != QKN_OK) return st;
    if (T == 0) return ok();
    qkn_launch L;
    if ((st = plan_call<qkn::kApply>(c, L)) != QKN_OK) return st;
    return launch<qkn::kApply>(c, L, stream);
}

qkn_status qknorm_combine_apply_launch(const void *q_in, void *q_out, const void *gamma_q_shard, int64_t q_stride,
                                       int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full,
                                       const void *k_in, void *k_out, const void *gamma_k_shard, int64_t k_stride,
                                       int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full,
                                       int32_t P, int64_t T, float eps, qkn_dtype dtype, void *stream,
                                       const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    Call c;
    qkn_status st = prepare_apply(q_in, q_out, gamma_q_shard, q_stride, hq_shard, q_sumsq_all, Hq_full, k_in, k_out,
                                  gamma_k_shard, k_stride, hk_shard, k_sumsq_all, Hk_full, P, T, eps, dtype, c);
    if (st != QKN_OK) return st;
    if ((st = check_launch<qkn::kApply>(c, *launch_cfg)) != QKN_OK) return st;
    if (T == 0) return ok();
    return launch<qkn::kApply>(c, *launch_cfg, stream);
}

}  // extern "C"

namespace {

qkn_status stats_shards(int32_t P, const void *const *q_shards, int64_t q_stride, int32_t hq_shard,
                        float *q_sumsq_all, const void *const *k_shards, int64_t k_stride, int32_t hk_shard,
                        float *k_sumsq_all, int64_t T, qkn_dtype dtype, void *stream, const qkn_launch *pinned) {
    ShardCall c;
    qkn_status st = prepare_stats_shards(P, q_shards, q_stride, hq_shard, q_sumsq_all, k_shards, k_stride, hk_shard,
                                         k_sumsq_all, T, dtype, c);
    if (st != QKN_OK) return st;
    if (pinned) {
        if (T > 0 && !one_launch(c))
            return fail(QKN_ERR_INVALID_ARG, "a pinned launch needs 16-byte aligned shard rows of at most 32 KB");
        if (T > 0 && (st = check_launch<qkn::kStats>(c, *pinned)) != QKN_OK) return st;
        if (T > 0 && pinned->kernel != QKN_KERNEL_REGISTER)
            return fail(QKN_ERR_INVALID_ARG, "multi-shard calls run the register kernel only");
        if (T == 0) return ok();
        return launch<qkn::kStats>(c, *pinned, stream);
    }
    if (T == 0) return ok();
    if (!one_launch(c)) {
        for (int p = 0; p < P; ++p)
            if ((st = qknorm_partial_stats(q_shards[p], q_stride, hq_shard, q_sumsq_all + (int64_t)p * T, k_shards[p],
                                           k_stride, hk_shard, k_sumsq_all + (int64_t)p * T, T, dtype, stream)) !=
                QKN_OK)
                return st;
        return ok();
    }
    qkn_launch L;
    if ((st = plan_call<qkn::kStats>(c, L)) != QKN_OK) return st;
    return launch<qkn::kStats>(c, L, stream);
}

qkn_status apply_shards(int32_t P, const void *const *q_in, void *const *q_out, const void *const *gamma_q_shards,
                        int64_t q_stride, int32_t hq_shard, const float *q_sumsq_all, int32_t Hq_full,
                        const void *const *k_in, void *const *k_out, const void *const *gamma_k_shards,
                        int64_t k_stride, int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full, int64_t T,
                        float eps, qkn_dtype dtype, void *stream, const qkn_launch *pinned) {
    ShardCall c;
    qkn_status st = prepare_apply_shards(P, q_in, q_out, gamma_q_shards, q_stride, hq_shard, q_sumsq_all, Hq_full,
                                         k_in, k_out, gamma_k_shards, k_stride, hk_shard, k_sumsq_all, Hk_full, T, eps,
                                         dtype, c);
    if (st != QKN_OK) return st;
    if (pinned) {
        if (T > 0 && !one_launch(c))
            return fail(QKN_ERR_INVALID_ARG, "a pinned launch needs 16-byte aligned shard rows of at most 32 KB");
        if (T > 0 && (st = check_launch<qkn::kApply>(c, *pinned)) != QKN_OK) return st;
        if (T > 0 && pinned->kernel != QKN_KERNEL_REGISTER)
            return fail(QKN_ERR_INVALID_ARG, "multi-shard calls run the register kernel only");
        if (T == 0) return ok();
        return launch<qkn::kApply>(c, *pinned, stream);
    }
    if (T == 0) return ok();
    if (!one_launch(c)) {
        for (int p = 0; p < P; ++p)
            if ((st = qknorm_combine_apply(q_in[p], q_out[p], gamma_q_shards[p], q_stride, hq_shard, q_sumsq_all,
                                           Hq_full, k_in[p], k_out[p], gamma_k_shards[p], k_stride, hk_shard,
                                           k_sumsq_all, Hk_full, P, T, eps, dtype, stream)) != QKN_OK)
                return st;
        return ok();
    }
    qkn_launch L;
    if ((st = plan_call<qkn::kApply>(c, L)) != QKN_OK) return st;
    return launch<qkn::kApply>(c, L, stream);
}

}  // namespace

extern "C" {

qkn_status qknorm_partial_stats_shards(int32_t P, const void *const *q_shards, int64_t q_stride, int32_t hq_shard,
                                       float *q_sumsq_all, const void *const *k_shards, int64_t k_stride,
                                       int32_t hk_shard, float *k_sumsq_all, int64_t T, qkn_dtype dtype,
                                       void *stream) {
    return stats_shards(P, q_shards, q_stride, hq_shard, q_sumsq_all, k_shards, k_stride, hk_shard, k_sumsq_all, T,
                        dtype, stream, nullptr);
}

qkn_status qknorm_partial_stats_shards_launch(int32_t P, const void *const *q_shards, int64_t q_stride,
                                              int32_t hq_shard, float *q_sumsq_all, const void *const *k_shards,
                                              int64_t k_stride, int32_t hk_shard, float *k_sumsq_all, int64_t T,
                                              qkn_dtype dtype, void *stream, const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    return stats_shards(P, q_shards, q_stride, hq_shard, q_sumsq_all, k_shards, k_stride, hk_shard, k_sumsq_all, T,
                        dtype, stream, launch_cfg);
}

qkn_status qknorm_combine_apply_shards(int32_t P, const void *const *q_in, void *const *q_out,
                                       const void *const *gamma_q_shards, int64_t q_stride, int32_t hq_shard,
                                       const float *q_sumsq_all, int32_t Hq_full, const void *const *k_in,
                                       void *const *k_out, const void *const *gamma_k_shards, int64_t k_stride,
                                       int32_t hk_shard, const float *k_sumsq_all, int32_t Hk_full, int64_t T,
                                       float eps, qkn_dtype dtype, void *stream) {
    return apply_shards(P, q_in, q_out, gamma_q_shards, q_stride, hq_shard, q_sumsq_all, Hq_full, k_in, k_out,
                        gamma_k_shards, k_stride, hk_shard, k_sumsq_all, Hk_full, T, eps, dtype, stream, nullptr);
}

qkn_status qknorm_combine_apply_shards_launch(int32_t P, const void *const *q_in, void *const *q_out,
                                              const void *const *gamma_q_shards, int64_t q_stride, int32_t hq_shard,
                                              const float *q_sumsq_all, int32_t Hq_full, const void *const *k_in,
                                              void *const *k_out, const void *const *gamma_k_shards,
                                              int64_t k_stride, int32_t hk_shard, const float *k_sumsq_all,
                                              int32_t Hk_full, int64_t T, float eps, qkn_dtype dtype, void *stream,
                                              const qkn_launch *launch_cfg) {
    if (!launch_cfg) return fail(QKN_ERR_INVALID_ARG, "null launch");
    return apply_shards(P, q_in, q_out, gamma_q_shards, q_stride, hq_shard, q_sumsq_all, Hq_full, k_in, k_out,
                        gamma_k_shards, k_stride, hk_shard, k_sumsq_all, Hk_full, T, eps, dtype, stream, launch_cfg);
}

qkn_status qknorm_qkv_gemm_stats(const void *x, int64_t x_stride, const void *w, int64_t w_stride, void *qkv,
                                 int64_t qkv_stride, int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv,
                                 float *q_sumsq_all, float *k_sumsq_all, qkn_dtype dtype, void *stream) {
    Projection pr;
    qkn_status st = prepare_projection(x, x_stride, w, w_stride, qkv, qkv_stride, T, D, Hq, Hk, Hv, dtype, pr);
    if (st != QKN_OK) return st;
    if (T == 0) return ok();
    if (!q_sumsq_all || !k_sumsq_all) return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if ((reinterpret_cast<uintptr_t>(q_sumsq_all) | reinterpret_cast<uintptr_t>(k_sumsq_all)) & 3u)
        return fail(QKN_ERR_INVALID_ARG, "partial sums must be 4-byte aligned");
    if ((st = check_projection_overlaps(pr, q_sumsq_all, k_sumsq_all, nullptr, nullptr)) != QKN_OK) return st;
    return launch_projection_gemm(pr, q_sumsq_all, k_sumsq_all, stream);
}

int64_t qknorm_qkv_projection_workspace_bytes(int64_t T, int32_t Hq, int32_t Hk) {
    if (T < 0 || Hq <= 0 || Hk <= 0 || Hq % kTileN || Hk % kTileN) return -1;
    // partial sums [Hq/256][T] and [Hk/256][T]
    return (int64_t)(Hq / kTileN + Hk / kTileN) * T * 4;
}

qkn_status qknorm_qkv_gemm_schedule(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, int32_t clusters,
                                    int64_t l2_bytes, qkn_gemm_schedule *out) {
    if (!out) return fail(QKN_ERR_INVALID_ARG, "null output");
    qkn_status st = check_gemm_shape(T, D, Hq, Hk, Hv);
    if (st != QKN_OK) return st;
    if (clusters < 1 || l2_bytes < 0) return fail(QKN_ERR_INVALID_ARG, "clusters must be >= 1 and l2_bytes >= 0");
    qkn::gemm::GemmParams gp{};
    gemm_tiles(T, D, Hq, Hk, Hv, gp);
    qkn::gemm::schedule_qkv_gemm(&gp, D, Hq + Hk + Hv, clusters, l2_bytes);
    fill_schedule(gp, clusters, out);
    return ok();
}

qkn_status qknorm_qkv_gemm_plan(int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, qkn_gemm_schedule *out) {
    if (!out) return fail(QKN_ERR_INVALID_ARG, "null output");
    qkn_status st = check_gemm_shape(T, D, Hq, Hk, Hv);
    if (st != QKN_OK) return st;
    int clusters = 0, dev = 0, l2 = 0;
    const char *what = "";
    cudaError_t e = qkn::gemm::qkv_gemm_clusters(&clusters, &what);
    if (e == cudaSuccess && (e = cudaGetDevice(&dev)) != cudaSuccess) what = "cudaGetDevice";
    if (e == cudaSuccess && (e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev)) != cudaSuccess)
        what = "cudaDeviceGetAttribute(L2 cache size)";
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "projection plan (%s): %s", what, cudaGetErrorString(e));
    return qknorm_qkv_gemm_schedule(T, D, Hq, Hk, Hv, clusters, l2, out);
}

qkn_status qknorm_qkv_projection(const void *x, int64_t x_stride, const void *w, int64_t w_stride, void *qkv,
                                 int64_t qkv_stride, const void *gamma_q, const void *gamma_k, int64_t T, int32_t D,
                                 int32_t Hq, int32_t Hk, int32_t Hv, float eps, void *workspace,
                                 int64_t workspace_bytes, qkn_dtype dtype, void *stream) {
    Projection pr;
    qkn_status st = prepare_projection(x, x_stride, w, w_stride, qkv, qkv_stride, T, D, Hq, Hk, Hv, dtype, pr);
    if (st != QKN_OK) return st;
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (T == 0) return ok();
    const int64_t need = qknorm_qkv_projection_workspace_bytes(T, Hq, Hk);
    if (!gamma_q || !gamma_k || !workspace) return fail(QKN_ERR_INVALID_ARG, "null pointer");
    if (workspace_bytes < need)
        return fail(QKN_ERR_INVALID_ARG, "workspace of %lld bytes, %lld needed", (long long)workspace_bytes,
                    (long long)need);
    if (reinterpret_cast<uintptr_t>(workspace) & 3u) return fail(QKN_ERR_INVALID_ARG, "workspace must be 4-byte aligned");
    float *q_sums = static_cast<float *>(workspace);
    float *k_sums = q_sums + (int64_t)(Hq / kTileN) * T;
    if ((st = check_projection_overlaps(pr, q_sums, k_sums, gamma_q, gamma_k)) != QKN_OK) return st;
    {
        const Region wsr = flat_region(workspace, need);
        if (overlap(wsr, rows_region(qkv, pr.N, qkv_stride, T, 2)) || overlap(wsr, rows_region(x, D, x_stride, T, 2)) ||
            overlap(wsr, rows_region(w, D, w_stride, pr.N, 2)) || overlap(wsr, flat_region(gamma_q, (int64_t)Hq * 2)) ||
            overlap(wsr, flat_region(gamma_k, (int64_t)Hk * 2)))
            return fail(QKN_ERR_INVALID_ARG, "the workspace overlaps an operand");
    }

    // The GEMM writes qkv and the partial sums; a second launch then runs
    // Phase A's aggregation and Phase B over the Q and K columns of qkv, in
    // place, while the freshly stored tiles are partly still in L2.  (Scaling
    // the tiles inside the GEMM's epilogue once a strip was complete gave the
    // same bits but was slower or equal: its read-modify-write competes with
    // the GEMM's operand stream.)
    Call c;
    init_call(c, dtype, 2);
    char *kcols = static_cast<char *>(qkv) + (int64_t)Hq * 2;
    fill_rowset(c.p.set[0], qkv, qkv, gamma_q, qkv_stride, Hq, Hq, 2);
    fill_rowset(c.p.set[1], kcols, kcols, gamma_k, qkv_stride, Hk, Hk, 2);
    c.p.set[0].sumsq_all = q_sums;
    c.p.set[1].sumsq_all = k_sums;
    c.p.set[0].P = Hq / kTileN;
    c.p.set[1].P = Hk / kTileN;
    c.p.T = T;
    c.p.eps = eps;
    finish_call(c, 2, {qkv, kcols, gamma_q, gamma_k}, qkv_stride, qkv_stride);
    qkn_launch L;
    if ((st = plan_call<qkn::kApply>(c, L)) != QKN_OK) return st;
    if ((st = launch_projection_gemm(pr, q_sums, k_sums, stream)) != QKN_OK) return st;
    return launch<qkn::kApply>(c, L, stream);
}

qkn_status qknorm_qkv_projection_noalloc(const void *x, int64_t x_stride, const void *w, int64_t w_stride,
                                         void *qkv, int64_t qkv_stride, const void *gamma_q, const void *gamma_k,
                                         int64_t T, int32_t D, int32_t Hq, int32_t Hk, int32_t Hv, float eps,
                                         qkn_dtype dtype, void *stream) {
    const int64_t need = qknorm_qkv_projection_workspace_bytes(T, Hq, Hk);
    if (T <= 0 || need < 0)  // empty or invalid: the checks below reject it or do nothing
        return qknorm_qkv_projection(x, x_stride, w, w_stride, qkv, qkv_stride, gamma_q, gamma_k, T, D, Hq, Hk, Hv,
                                     eps, nullptr, 0, dtype, stream);
    if (need > kNoAllocScratchBytes)
        return fail(QKN_ERR_INVALID_ARG,
                    "needs %lld bytes of workspace for the partial sums; the built-in scratch holds %lld",
                    (long long)need, (long long)kNoAllocScratchBytes);
    void *ws = nullptr;
    qkn_status st = noalloc_scratch(&ws);
    if (st != QKN_OK) return st;
    return qknorm_qkv_projection(x, x_stride, w, w_stride, qkv, qkv_stride, gamma_q, gamma_k, T, D, Hq, Hk, Hv, eps,
                                 ws, kNoAllocScratchBytes, dtype, stream);
}

int64_t qknorm_qkv_projection_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

qkn_status qknorm_device_timeouts(int32_t *code) {
    if (!code) return fail(QKN_ERR_INVALID_ARG, "null pointer");
    int v = 0, w = 0;
    cudaError_t e = qkn::gemm::read_and_clear_timeout(&v);
    if (e == cudaSuccess) e = qkn::tp::tp_read_and_clear_timeout(&w);
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "reading the timeout word: %s", cudaGetErrorString(e));
    *code = v ? v : w;
    return ok();
}

int64_t qknorm_tp_recv_bytes(int32_t R, int64_t T) {
    if (R < 1 || R > qkn::tp::kMaxRanks || T < 0 || T >= ((int64_t)1 << 31)) return -1;
    return (int64_t)R * T * 2 * 8 + 16;  // exchange words, then the 16-byte trailer (abort word)
}

}  // extern "C"

namespace {

// qknorm_tp_layerwise with the exchange scope: scope 0 picks GPU scope when
// every rank of the group runs in the call and system scope otherwise; scope 1
// takes system scope whatever runs where.
qkn_status tp_layerwise(int32_t R, int32_t first_rank, int32_t n_local, const void *const *q_in,
                        void *const *q_out, const void *const *gamma_q, int64_t q_stride, int32_t hq_shard,
                        int32_t Hq_full, const void *const *k_in, void *const *k_out, const void *const *gamma_k,
                        int64_t k_stride, int32_t hk_shard, int32_t Hk_full, int64_t T, float eps, qkn_dtype dtype,
                        void *const *recv, uint32_t epoch, int32_t blocks_per_rank, uint64_t timeout_ns,
                        int32_t scope, void *stream) {
    using qkn::tp::kMaxLocal;
    using qkn::tp::kMaxRanks;
    if (scope != 0 && scope != 1) return fail(QKN_ERR_INVALID_ARG, "scope must be 0 (automatic) or 1 (system)");
    if (!dtype_valid(dtype)) return fail(QKN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (R < 1 || R > kMaxRanks) return fail(QKN_ERR_INVALID_ARG, "R = %d outside [1, %d]", R, kMaxRanks);
    if (n_local < 1 || n_local > kMaxLocal || first_rank < 0 || first_rank + n_local > R)
        return fail(QKN_ERR_INVALID_ARG, "local ranks [%d, %d) outside [0, %d)", first_rank, first_rank + n_local, R);
    if (T < 0 || T >= ((int64_t)1 << 31)) return fail(QKN_ERR_INVALID_ARG, "T must be in [0, 2^31)");
    if (hq_shard <= 0 || hk_shard <= 0) return fail(QKN_ERR_INVALID_ARG, "shard widths must be positive");
    if (Hq_full < hq_shard || Hk_full < hk_shard) return fail(QKN_ERR_INVALID_ARG, "full width below shard width");
    if (q_stride < hq_shard || k_stride < hk_shard) return fail(QKN_ERR_INVALID_ARG, "row stride below shard width");
    if (!eps_valid(eps)) return fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (epoch == 0) return fail(QKN_ERR_INVALID_ARG, "epoch 0 is reserved (receive buffers start zeroed)");
    if (blocks_per_rank < 0) return fail(QKN_ERR_INVALID_ARG, "blocks_per_rank < 0");
    const int esz = elem_bytes(dtype);
    if (!extent_ok(T, q_stride, hq_shard, esz) || !extent_ok(T, k_stride, hk_shard, esz))
        return fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T == 0) return ok();
    if (!q_in || !q_out || !gamma_q || !k_in || !k_out || !gamma_k || !recv)
        return fail(QKN_ERR_INVALID_ARG, "null pointer array");
    for (int r = 0; r < R; ++r)
        if (!recv[r] || (reinterpret_cast<uintptr_t>(recv[r]) & 15u))
            return fail(QKN_ERR_INVALID_ARG, "receive buffer %d null or not 16-byte aligned", r);
    const int per_vec = 16 / esz;
    if (hq_shard % per_vec || hk_shard % per_vec || (q_stride * esz) % 16 || (k_stride * esz) % 16)
        return fail(QKN_ERR_UNSUPPORTED, "shard widths and strides must be whole 16-byte vectors");
    const int gsz = gamma_bytes(dtype);
    for (int j = 0; j < n_local; ++j) {
        const void *ptrs[6] = {q_in[j], q_out[j], gamma_q[j], k_in[j], k_out[j], gamma_k[j]};
        for (const void *pp : ptrs)
            if (!pp) return fail(QKN_ERR_INVALID_ARG, "null pointer for local rank %d", j);
            else if (!aligned16(pp)) return fail(QKN_ERR_UNSUPPORTED, "local rank %d: buffers must be 16-byte aligned", j);
        const Region iq = rows_region(q_in[j], hq_shard, q_stride, T, esz), oq = rows_region(q_out[j], hq_shard, q_stride, T, esz);
        const Region ik = rows_region(k_in[j], hk_shard, k_stride, T, esz), ok_ = rows_region(k_out[j], hk_shard, k_stride, T, esz);
        const Region others[2] = {flat_region(gamma_q[j], (int64_t)hq_shard * gsz),
                                  flat_region(gamma_k[j], (int64_t)hk_shard * gsz)};
        qkn_status st = check_outputs(oq, ok_, iq, ik, others, 2);
        if (st != QKN_OK) return st;
        // the kernel writes every rank's receive buffer: none may share a byte
        // with this rank's rows or gamma slices
        for (int r = 0; r < R; ++r) {
            const Region rb = flat_region(recv[r], qknorm_tp_recv_bytes(R, T));
            if (overlap(rb, oq) || overlap(rb, ok_) || overlap(rb, iq) || overlap(rb, ik) || overlap(rb, others[0]) ||
                overlap(rb, others[1]))
                return fail(QKN_ERR_INVALID_ARG, "receive buffer %d overlaps local rank %d's rows or gamma", r, j);
        }
    }
    for (int r = 0; r < R; ++r)  // nor one another
        for (int r2 = r + 1; r2 < R; ++r2)
            if (overlap(flat_region(recv[r], qknorm_tp_recv_bytes(R, T)), flat_region(recv[r2], qknorm_tp_recv_bytes(R, T))))
                return fail(QKN_ERR_INVALID_ARG, "receive buffers %d and %d overlap", r, r2);
    for (int j = 0; j < n_local; ++j)  // no rank's output may touch another local rank's buffers
        for (int jj = 0; jj < n_local; ++jj) {
            if (jj == j) continue;
            const Region outs[2] = {rows_region(q_out[j], hq_shard, q_stride, T, esz),
                                    rows_region(k_out[j], hk_shard, k_stride, T, esz)};
            const Region theirs[4] = {rows_region(q_in[jj], hq_shard, q_stride, T, esz),
                                      rows_region(k_in[jj], hk_shard, k_stride, T, esz),
                                      rows_region(q_out[jj], hq_shard, q_stride, T, esz),
                                      rows_region(k_out[jj], hk_shard, k_stride, T, esz)};
            for (const Region &o : outs)
                for (const Region &t : theirs)
                    if (overlap(o, t)) return fail(QKN_ERR_INVALID_ARG, "rank %d's output overlaps rank %d's rows", j, jj);
        }
    // launch shape: one token per warp, four warps per block; rows of up to 8
    // vectors per lane unrolled, wider ones in a batch loop
    const int64_t vq = hq_shard / per_vec, vk = hk_shard / per_vec, vmax = vq > vk ? vq : vk;
    int nv = 0;
    const int threads = 128;
    const int64_t tokens_per_block = 4;
    if (vmax <= 256) {
        auto lanes_nv = [](int64_t v) { return v <= 32 ? 1 : (v <= 64 ? 2 : (v <= 128 ? 4 : 8)); };
        int nvq = lanes_nv(vq), nvk = lanes_nv(vk);
        if (nvk > nvq) nvq = nvk;  // instantiated with NVK <= NVQ
        nv = -(8 * nvq + nvk);
    }
    int dev = 0, sms = 0, bps = 0;
    qkn_status st = current_device(&dev);
    if (st != QKN_OK) return st;
    if ((st = sm_count(dev, &sms)) != QKN_OK) return st;
    const bool gpu_scope = n_local == R && scope == 0;
    cudaError_t e = qkn::tp::tp_blocks_per_sm((int)dtype, nv, threads, gpu_scope, &bps);
    if (e != cudaSuccess || bps < 1) return fail(QKN_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    const int64_t resident = (int64_t)bps * sms;
    int64_t G = blocks_per_rank > 0 ? blocks_per_rank : resident / n_local;
    const int64_t needed = (T + tokens_per_block - 1) / tokens_per_block;
    if (G > needed) G = needed;
    if (G < 1 || G * n_local > resident)
        return fail(QKN_ERR_UNSUPPORTED, "%lld blocks per rank x %d ranks exceed the %lld resident blocks",
                    (long long)G, n_local, (long long)resident);
    qkn::tp::TpParams tp{};
    for (int j = 0; j < n_local; ++j)
        tp.local[j] = qkn::tp::RankPtrs{static_cast<const char *>(q_in[j]), static_cast<char *>(q_out[j]),
                                        static_cast<const char *>(gamma_q[j]), static_cast<const char *>(k_in[j]),
                                        static_cast<char *>(k_out[j]), static_cast<const char *>(gamma_k[j])};
    for (int r = 0; r < R; ++r) tp.recv[r] = static_cast<unsigned long long *>(recv[r]);
    tp.q_stride_bytes = q_stride * esz;
    tp.k_stride_bytes = k_stride * esz;
    tp.T = T;
    tp.R = R;
    tp.first_rank = first_rank;
    tp.n_local = n_local;
    tp.blocks_per_rank = (int32_t)G;
    tp.q_vecs = (int32_t)vq;
    tp.k_vecs = (int32_t)vk;
    tp.inv_hq = static_cast<float>(1.0 / static_cast<double>(Hq_full));
    tp.inv_hk = static_cast<float>(1.0 / static_cast<double>(Hk_full));
    tp.eps = eps;
    tp.epoch = epoch;
    tp.timeout_ns = timeout_ns ? timeout_ns : kGemmTimeoutNs;
    const char *what = "";
    e = qkn::tp::launch_tp(tp, (int)dtype, nv, threads, gpu_scope, static_cast<cudaStream_t>(stream), &what);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(QKN_ERR_CUDA, "tensor-parallel kernel (%s): %s", what, cudaGetErrorString(e));
    return ok();
}

}  // namespace

extern "C" {

qkn_status qknorm_tp_layerwise(int32_t R, int32_t first_rank, int32_t n_local, const void *const *q_in,
                               void *const *q_out, const void *const *gamma_q, int64_t q_stride, int32_t hq_shard,
                               int32_t Hq_full, const void *const *k_in, void *const *k_out,
                               const void *const *gamma_k, int64_t k_stride, int32_t hk_shard, int32_t Hk_full,
                               int64_t T, float eps, qkn_dtype dtype, void *const *recv, uint32_t epoch,
                               int32_t blocks_per_rank, uint64_t timeout_ns, void *stream) {
    return tp_layerwise(R, first_rank, n_local, q_in, q_out, gamma_q, q_stride, hq_shard, Hq_full, k_in, k_out,
                        gamma_k, k_stride, hk_shard, Hk_full, T, eps, dtype, recv, epoch, blocks_per_rank, timeout_ns,
                        0, stream);
}

qkn_status qknorm_tp_layerwise_scope(int32_t R, int32_t first_rank, int32_t n_local, const void *const *q_in,
                                     void *const *q_out, const void *const *gamma_q, int64_t q_stride,
                                     int32_t hq_shard, int32_t Hq_full, const void *const *k_in, void *const *k_out,
                                     const void *const *gamma_k, int64_t k_stride, int32_t hk_shard, int32_t Hk_full,
                                     int64_t T, float eps, qkn_dtype dtype, void *const *recv, uint32_t epoch,
                                     int32_t blocks_per_rank, uint64_t timeout_ns, int32_t scope, void *stream) {
    return tp_layerwise(R, first_rank, n_local, q_in, q_out, gamma_q, q_stride, hq_shard, Hq_full, k_in, k_out,
                        gamma_k, k_stride, hk_shard, Hk_full, T, eps, dtype, recv, epoch, blocks_per_rank, timeout_ns,
                        scope, stream);
}

const char *qknorm_status_string(qkn_status s) {
    switch (s) {
        case QKN_OK: return "ok";
        case QKN_ERR_INVALID_ARG: return "invalid argument";
        case QKN_ERR_MISALIGNED: return "misaligned (reserved; not returned)";
        case QKN_ERR_UNSUPPORTED: return "unsupported";
        case QKN_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

const char *qknorm_last_error(void) { return g_last_error; }

int qknorm_version(void) { return QKNORM_VERSION; }

}  // extern "C"
