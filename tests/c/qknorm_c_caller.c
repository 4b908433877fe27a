/*
 * A plain C caller of libqknorm.so: no Python, no torch.  Reads Q, K and the
 * two gamma vectors (bfloat16 bits) from files, normalizes them on the GPU
 * through the C ABI twice, and writes both results:
 *   - qknorm_layerwise on device buffers -> qo.bin, ko.bin;
 *   - qknorm_layerwise_host on page-locked host buffers, in place, in chunks
 *     of `chunk` tokens through a two-slot device ring on three streams ->
 *     qo_host.bin, ko_host.bin.
 *
 *   qknorm_c_caller T Hq Hk eps chunk q.bin k.bin gq.bin gk.bin qo.bin ko.bin qo_host.bin ko_host.bin
 *
 * Exit status 0 on success; any CUDA or library error is printed with the
 * library's own message.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "qknorm.h"

static void *read_file(const char *path, size_t bytes) {
    FILE *f = fopen(path, "rb");
    if (!f) return NULL;
    void *buf = malloc(bytes ? bytes : 1);
    size_t got = fread(buf, 1, bytes, f);
    fclose(f);
    if (got != bytes) {
        free(buf);
        return NULL;
    }
    return buf;
}

static int write_file(const char *path, const void *buf, size_t bytes) {
    FILE *f = fopen(path, "wb");
    if (!f) return -1;
    size_t put = fwrite(buf, 1, bytes, f);
    fclose(f);
    return put == bytes ? 0 : -1;
}

#define CHECK_CUDA(call)                                                              \
    do {                                                                              \
        cudaError_t e_ = (call);                                                      \
        if (e_ != cudaSuccess) {                                                      \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));               \
            return 2;                                                                 \
        }                                                                             \
    } while (0)

int main(int argc, char **argv) {
    if (argc != 14) {
        fprintf(stderr, "usage: %s T Hq Hk eps chunk q k gq gk qo ko qo_host ko_host\n", argv[0]);
        return 1;
    }
    const long long T = atoll(argv[1]);
    const int Hq = atoi(argv[2]), Hk = atoi(argv[3]);
    const float eps = (float)atof(argv[4]);
    const long long chunk = atoll(argv[5]);
    const size_t qb = (size_t)T * Hq * 2, kb = (size_t)T * Hk * 2;
    void *hq = read_file(argv[6], qb), *hk = read_file(argv[7], kb);
    void *hgq = read_file(argv[8], (size_t)Hq * 2), *hgk = read_file(argv[9], (size_t)Hk * 2);
    if (!hq || !hk || !hgq || !hgk) {
        fprintf(stderr, "could not read the inputs\n");
        return 1;
    }
    printf("library version %d\n", qknorm_version());

    void *dq, *dk, *dgq, *dgk, *dqo, *dko;
    CHECK_CUDA(cudaMalloc(&dq, qb));
    CHECK_CUDA(cudaMalloc(&dk, kb));
    CHECK_CUDA(cudaMalloc(&dgq, (size_t)Hq * 2));
    CHECK_CUDA(cudaMalloc(&dgk, (size_t)Hk * 2));
    CHECK_CUDA(cudaMalloc(&dqo, qb));
    CHECK_CUDA(cudaMalloc(&dko, kb));
    CHECK_CUDA(cudaMemcpy(dq, hq, qb, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(dk, hk, kb, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(dgq, hgq, (size_t)Hq * 2, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(dgk, hgk, (size_t)Hk * 2, cudaMemcpyHostToDevice));

    /* a rejected call says why and enqueues nothing */
    qkn_status bad = qknorm_layerwise(dq, dqo, dgq, Hq, dk, dko, dgk, Hk, T, Hq, Hk, -1.0f, QKN_BF16, NULL);
    printf("negative eps: %s (%s)\n", qknorm_status_string(bad), qknorm_last_error());
    if (bad != QKN_ERR_INVALID_ARG) return 3;

    cudaStream_t s;
    CHECK_CUDA(cudaStreamCreate(&s));
    qkn_status st = qknorm_layerwise(dq, dqo, dgq, Hq, dk, dko, dgk, Hk, T, Hq, Hk, eps, QKN_BF16, (void *)s);
    if (st != QKN_OK) {
        fprintf(stderr, "qknorm_layerwise: %s: %s\n", qknorm_status_string(st), qknorm_last_error());
        return 4;
    }
    CHECK_CUDA(cudaStreamSynchronize(s));

    /* the same rows from page-locked host memory, normalized in place */
    void *pq, *pk;
    CHECK_CUDA(cudaHostAlloc(&pq, qb, cudaHostAllocDefault));
    CHECK_CUDA(cudaHostAlloc(&pk, kb, cudaHostAllocDefault));
    memcpy(pq, hq, qb);
    memcpy(pk, hk, kb);
    const int64_t ring_bytes = qknorm_layerwise_host_ring_bytes(chunk, Hq, Hk, QKN_BF16, 2);
    if (ring_bytes < 0) {
        fprintf(stderr, "qknorm_layerwise_host_ring_bytes refused chunk %lld\n", chunk);
        return 5;
    }
    void *ring;
    CHECK_CUDA(cudaMalloc(&ring, (size_t)ring_bytes));
    cudaStream_t s_in, s_out;
    CHECK_CUDA(cudaStreamCreate(&s_in));
    CHECK_CUDA(cudaStreamCreate(&s_out));
    st = qknorm_layerwise_host(pq, pq, dgq, Hq, pk, pk, dgk, Hk, T, Hq, Hk, eps, QKN_BF16, ring, ring_bytes, chunk,
                               (void *)s, (void *)s_in, (void *)s_out);
    if (st != QKN_OK) {
        fprintf(stderr, "qknorm_layerwise_host: %s: %s\n", qknorm_status_string(st), qknorm_last_error());
        return 6;
    }
    CHECK_CUDA(cudaStreamSynchronize(s)); /* the call is complete once `s` passes it */

    CHECK_CUDA(cudaMemcpy(hq, dqo, qb, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(hk, dko, kb, cudaMemcpyDeviceToHost));
    if (write_file(argv[10], hq, qb) || write_file(argv[11], hk, kb) || write_file(argv[12], pq, qb) ||
        write_file(argv[13], pk, kb)) {
        fprintf(stderr, "could not write the outputs\n");
        return 1;
    }
    cudaStreamDestroy(s_in);
    cudaStreamDestroy(s_out);
    cudaFree(ring);
    cudaFreeHost(pq);
    cudaFreeHost(pk);
    cudaStreamDestroy(s);
    cudaFree(dq);
    cudaFree(dk);
    cudaFree(dgq);
    cudaFree(dgk);
    cudaFree(dqo);
    cudaFree(dko);
    printf("ok\n");
    return 0;
}
