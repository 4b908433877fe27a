// Layerwise QK-Norm on rows held in host memory (qknorm_layerwise_host in
// include/qknorm.h): the batch flows in chunks of tokens through a ring of
// caller-owned device buffers on three streams, so that the host->device copy
// of one chunk, the normalization of the previous one (qknorm_layerwise on the
// device copy, in place) and the device->host copy of the one before overlap.
// Only host code: it enqueues copies, kernel launches and event waits; every
// element is normalized by the library's kernel.
//
// Per chunk i in ring slot s = i mod slots:
//   copy_in  : waits freed[s] (chunk i - slots copied out), copies Q and K
//              rows host->device, records loaded[s];
//   stream   : waits loaded[s], normalizes in place, records computed[s];
//   copy_out : waits computed[s], copies the rows device->host, records freed[s].
// An event is recorded again only after every wait on its previous record has
// been enqueued (cudaStreamWaitEvent takes the record current at the time of
// the call), so one set of 3 * slots events serves any number of chunks.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

#include "qknorm.h"
#include "qknorm_plan.h"

namespace qkn {
void set_last_error(const char *msg);  // qknorm_api.cu: the message qknorm_last_error returns
}  // namespace qkn

namespace {

constexpr int64_t kAlign = 256;

int64_t round_up(int64_t n, int64_t a) { return (n + a - 1) / a * a; }

int elem_size(qkn_dtype dt) { return dt == QKN_F32 ? 4 : (dt == QKN_FP8_E4M3 ? 1 : 2); }

// Bytes of one ring slot: chunk_tokens rows of Q, then of K, each part
// starting on a 256-byte boundary.
int64_t slot_bytes(int64_t chunk_tokens, int32_t Hq, int32_t Hk, int esz) {
    return round_up(chunk_tokens * Hq * esz, kAlign) + round_up(chunk_tokens * Hk * esz, kAlign);
}

qkn_status host_fail(qkn_status st, const char *msg, cudaError_t e = cudaSuccess) {
    char buf[512];
    if (e != cudaSuccess)
        snprintf(buf, sizeof(buf), "%s: %s", msg, cudaGetErrorString(e));
    else
        snprintf(buf, sizeof(buf), "%s", msg);
    qkn::set_last_error(buf);
    return st;
}

// `rows` rows of `width_bytes` between a strided host matrix and contiguous
// device rows: one copy per call (a plain copy when the host rows are
// contiguous, else a pitched one).
cudaError_t copy_rows(void *dst, int64_t dpitch, const void *src, int64_t spitch, int64_t width_bytes, int64_t rows,
                      cudaMemcpyKind kind, cudaStream_t s) {
    if (dpitch == width_bytes && spitch == width_bytes)
        return cudaMemcpyAsync(dst, src, (size_t)(width_bytes * rows), kind, s);
    return cudaMemcpy2DAsync(dst, (size_t)dpitch, src, (size_t)spitch, (size_t)width_bytes, (size_t)rows, kind, s);
}

struct Events {
    cudaEvent_t start = nullptr;
    cudaEvent_t loaded[QKN_HOST_MAX_SLOTS] = {};
    cudaEvent_t computed[QKN_HOST_MAX_SLOTS] = {};
    cudaEvent_t freed[QKN_HOST_MAX_SLOTS] = {};
    int n = 0;

    cudaError_t create(int slots) {
        n = slots;
        cudaError_t e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
        for (int i = 0; i < slots && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&loaded[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&computed[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&freed[i], cudaEventDisableTiming);
        }
        return e;
    }
    // Destroying an event whose record has not completed is allowed: its
    // resources are released once it completes.
    ~Events() {
        if (start) cudaEventDestroy(start);
        for (int i = 0; i < n; ++i) {
            if (loaded[i]) cudaEventDestroy(loaded[i]);
            if (computed[i]) cudaEventDestroy(computed[i]);
            if (freed[i]) cudaEventDestroy(freed[i]);
        }
    }
};

bool overlaps(const void *a, int64_t aw, int64_t as, int64_t ar, const void *b, int64_t bw, int64_t bs, int64_t br) {
    return qknorm_regions_overlap((uint64_t)(uintptr_t)a, aw, as, ar, (uint64_t)(uintptr_t)b, bw, bs, br) != 0;
}

}  // namespace

extern "C" {

int64_t qknorm_layerwise_host_ring_bytes(int64_t chunk_tokens, int32_t Hq, int32_t Hk, qkn_dtype dtype,
                                         int32_t slots) {
    if (chunk_tokens < 1 || Hq < 1 || Hk < 1 || slots < 1 || slots > QKN_HOST_MAX_SLOTS) return -1;
    if (dtype < QKN_F32 || dtype > QKN_FP8_E4M3) return -1;
    if (chunk_tokens > ((int64_t)1 << 31)) return -1;
    return (int64_t)slots * slot_bytes(chunk_tokens, Hq, Hk, elem_size(dtype));
}

qkn_status qknorm_layerwise_host(const void *q_in, void *q_out, const void *gamma_q, int64_t q_stride,
                                 const void *k_in, void *k_out, const void *gamma_k, int64_t k_stride,
                                 int64_t T, int32_t Hq, int32_t Hk, float eps, qkn_dtype dtype, void *ring,
                                 int64_t ring_bytes, int64_t chunk_tokens, void *stream, void *copy_in_stream,
                                 void *copy_out_stream) {
    qkn::set_last_error("");
    if (dtype < QKN_F32 || dtype > QKN_FP8_E4M3) return host_fail(QKN_ERR_INVALID_ARG, "unknown dtype");
    if (T < 0) return host_fail(QKN_ERR_INVALID_ARG, "T < 0");
    if (Hq < 1 || Hk < 1) return host_fail(QKN_ERR_INVALID_ARG, "widths must be positive");
    if (q_stride < Hq || k_stride < Hk) return host_fail(QKN_ERR_INVALID_ARG, "row stride below width");
    if (!std::isfinite(eps) || eps < 0.0f) return host_fail(QKN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (chunk_tokens < 1) return host_fail(QKN_ERR_INVALID_ARG, "chunk_tokens must be >= 1");
    const int esz = elem_size(dtype);
    if (T > 0 && ((__int128)(T - 1) * (q_stride > k_stride ? q_stride : k_stride) + (Hq > Hk ? Hq : Hk)) * esz >=
                     ((__int128)1 << 62))
        return host_fail(QKN_ERR_INVALID_ARG, "buffer extent overflows");
    if (T == 0) return QKN_OK;
    if (!q_in || !q_out || !k_in || !k_out || !gamma_q || !gamma_k || !ring)
        return host_fail(QKN_ERR_INVALID_ARG, "null pointer");
    const int64_t chunk = chunk_tokens < T ? chunk_tokens : T;
    const int64_t per_slot = slot_bytes(chunk, Hq, Hk, esz);
    if (ring_bytes < per_slot)
        return host_fail(QKN_ERR_INVALID_ARG, "ring smaller than one slot (qknorm_layerwise_host_ring_bytes)");
    if (reinterpret_cast<uintptr_t>(ring) % kAlign) return host_fail(QKN_ERR_INVALID_ARG, "ring must be 256-byte aligned");
    int64_t slots = ring_bytes / per_slot;
    if (slots > QKN_HOST_MAX_SLOTS) slots = QKN_HOST_MAX_SLOTS;

    // host regions: outputs may equal their inputs (in place) and nothing else
    const int64_t qw = (int64_t)Hq * esz, kw = (int64_t)Hk * esz, qs = q_stride * esz, ks = k_stride * esz;
    if (overlaps(q_out, qw, qs, T, k_out, kw, ks, T)) return host_fail(QKN_ERR_INVALID_ARG, "q_out and k_out overlap");
    if (q_out != q_in && overlaps(q_out, qw, qs, T, q_in, qw, qs, T))
        return host_fail(QKN_ERR_INVALID_ARG, "q_out partly overlaps q_in (only out == in is allowed)");
    if (k_out != k_in && overlaps(k_out, kw, ks, T, k_in, kw, ks, T))
        return host_fail(QKN_ERR_INVALID_ARG, "k_out partly overlaps k_in (only out == in is allowed)");
    if (overlaps(q_out, qw, qs, T, k_in, kw, ks, T) || overlaps(k_out, kw, ks, T, q_in, qw, qs, T))
        return host_fail(QKN_ERR_INVALID_ARG, "an output overlaps the other tensor's input");
    const int64_t gsz = dtype == QKN_F32 ? 4 : 2;
    const int64_t ring_used = slots * per_slot;
    if (overlaps(ring, ring_used, ring_used, 1, gamma_q, Hq * gsz, Hq * gsz, 1) ||
        overlaps(ring, ring_used, ring_used, 1, gamma_k, Hk * gsz, Hk * gsz, 1))
        return host_fail(QKN_ERR_INVALID_ARG, "the ring overlaps gamma");

    cudaStream_t s_main = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = static_cast<cudaStream_t>(copy_in_stream);
    cudaStream_t s_out = static_cast<cudaStream_t>(copy_out_stream);
    Events ev;
    cudaError_t e = ev.create((int)slots);
    if (e != cudaSuccess) return host_fail(QKN_ERR_CUDA, "cudaEventCreateWithFlags", e);
    // everything the caller queued on `stream` before this call (gamma, an
    // earlier call on the same ring) comes first
    if ((e = cudaEventRecord(ev.start, s_main)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s_in, ev.start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s_out, ev.start, 0)) != cudaSuccess)
        return host_fail(QKN_ERR_CUDA, "ordering the copy streams after the stream", e);

    char *base = static_cast<char *>(ring);
    const char *qi = static_cast<const char *>(q_in), *ki = static_cast<const char *>(k_in);
    char *qo = static_cast<char *>(q_out), *ko = static_cast<char *>(k_out);
    const int64_t q_part = round_up(chunk * qw, kAlign);
    int64_t i = 0;
    for (int64_t t0 = 0; t0 < T; t0 += chunk, ++i) {
        const int64_t rows = T - t0 < chunk ? T - t0 : chunk;
        const int s = (int)(i % slots);
        char *dq = base + s * per_slot, *dk = dq + q_part;
        if (i >= slots && (e = cudaStreamWaitEvent(s_in, ev.freed[s], 0)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "copy-in wait", e);
        if ((e = copy_rows(dq, qw, qi + t0 * qs, qs, qw, rows, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
            (e = copy_rows(dk, kw, ki + t0 * ks, ks, kw, rows, cudaMemcpyHostToDevice, s_in)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "host->device copy", e);
        if ((e = cudaEventRecord(ev.loaded[s], s_in)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(s_main, ev.loaded[s], 0)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "ordering the kernel after its copy", e);
        const qkn_status st = qknorm_layerwise(dq, dq, gamma_q, Hq, dk, dk, gamma_k, Hk, rows, Hq, Hk, eps, dtype,
                                               stream);
        if (st != QKN_OK) {
            char buf[512];
            snprintf(buf, sizeof(buf), "qknorm_layerwise on chunk %lld: %s", (long long)i, qknorm_last_error());
            qkn::set_last_error(buf);
            return st;
        }
        if ((e = cudaEventRecord(ev.computed[s], s_main)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(s_out, ev.computed[s], 0)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "ordering the copy back after the kernel", e);
        if ((e = copy_rows(qo + t0 * qs, qs, dq, qw, qw, rows, cudaMemcpyDeviceToHost, s_out)) != cudaSuccess ||
            (e = copy_rows(ko + t0 * ks, ks, dk, kw, kw, rows, cudaMemcpyDeviceToHost, s_out)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "device->host copy", e);
        if ((e = cudaEventRecord(ev.freed[s], s_out)) != cudaSuccess)
            return host_fail(QKN_ERR_CUDA, "cudaEventRecord", e);
    }
    // the call is complete when `stream` passes this point
    if ((e = cudaStreamWaitEvent(s_main, ev.freed[(int)((i - 1) % slots)], 0)) != cudaSuccess)
        return host_fail(QKN_ERR_CUDA, "ordering the stream after the last copy back", e);
    return QKN_OK;
}

}  // extern "C"
