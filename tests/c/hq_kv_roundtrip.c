/* A C program that drives a compressed KV cache through libhq.so with include/hq.h
 * alone (plus the CUDA runtime for device memory): a dense rotation read from a
 * file, subtractive dither and a second Rice parameter for the halved symbol; two
 * appends, a read of every token in fp32, and the library's own Haar draw for the
 * seed.  Writes the stream, the offsets, the read and the drawn rotation to files
 * for the test that drives it to compare with the oracle.
 *
 *   hq_kv_roundtrip IN.bin Q.bin HEADS T1 T2 ALPHA K DK SEED OUTPREFIX
 *
 * IN.bin holds HEADS x (T1 + T2) x 128 bf16 values (uint16, head-major, one token's
 * 128 values contiguous); Q.bin a 128 x 128 fp32 orthogonal matrix, row-major.
 * Exit status 0 on success; messages on stderr. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "hq.h"

#define CK(x)                                                                        \
    do {                                                                             \
        cudaError_t e_ = (x);                                                        \
        if (e_ != cudaSuccess) {                                                     \
            fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, cudaGetErrorString(e_)); \
            return 2;                                                                \
        }                                                                            \
    } while (0)
#define HQ(x)                                                                        \
    do {                                                                             \
        int r_ = (x);                                                                \
        if (r_ != HQ_OK) {                                                           \
            fprintf(stderr, "%s:%d %s (%d)\n", __FILE__, __LINE__, hq_status_string(r_), r_); \
            return 3;                                                                \
        }                                                                            \
    } while (0)

static int read_file(const char *path, void *p, size_t n) {
    FILE *f = fopen(path, "rb");
    if (!f) return 1;
    const size_t got = fread(p, 1, n, f);
    fclose(f);
    return got != n;
}

static int write_file(const char *prefix, const char *name, const void *p, size_t n) {
    char path[1024];
    snprintf(path, sizeof path, "%s%s", prefix, name);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(p, 1, n, f) != n) return 1;
    return fclose(f) != 0;
}

int main(int argc, char **argv) {
    if (argc != 11) {
        fprintf(stderr, "usage: %s IN.bin Q.bin HEADS T1 T2 ALPHA K DK SEED OUTPREFIX\n", argv[0]);
        return 1;
    }
    const int32_t heads = atoi(argv[3]);
    const int64_t t1 = atoll(argv[4]), t2 = atoll(argv[5]), tokens = t1 + t2;
    const float alpha = (float)atof(argv[6]);
    const char *prefix = argv[10];
    if (hq_device_check() != HQ_OK) {
        fprintf(stderr, "no sm_100 device\n");
        return 4;
    }
    const size_t n = (size_t)heads * (size_t)tokens * 128;
    uint16_t *h_kv = malloc(n * 2);
    float *h_q = malloc(128 * 128 * 4);
    if (!h_kv || !h_q || read_file(argv[1], h_kv, n * 2) || read_file(argv[2], h_q, 128 * 128 * 4)) return 5;

    /* buffers: a stream of 16 bits per scalar, offsets and table rows for both appends */
    const uint64_t max_chunks = (uint64_t)heads * (uint64_t)((t1 + 31) / 32 + (t2 + 31) / 32);
    const uint64_t cap = (uint64_t)n / 2 + max_chunks * 64 + 1024;
    const int64_t tmax = t1 > t2 ? t1 : t2;
    size_t ws_bytes = 0;
    HQ(hq_workspace_bytes((uint64_t)heads * (uint64_t)((tmax + 31) / 32), &ws_bytes));
    void *d_kv, *d_ws;
    float *d_q, *d_qdraw, *d_out;
    uint32_t *d_words;
    uint64_t *d_offsets, *d_tail;
    hq_kv_append_row *d_table;
    hq_stats *d_stats;
    CK(cudaMalloc(&d_kv, n * 2));
    CK(cudaMalloc((void **)&d_q, 128 * 128 * 4));
    CK(cudaMalloc((void **)&d_qdraw, 128 * 128 * 4));
    CK(cudaMalloc((void **)&d_out, n * 4));
    CK(cudaMalloc((void **)&d_words, cap * 4));
    CK(cudaMalloc((void **)&d_offsets, (max_chunks + 1) * 8));
    CK(cudaMalloc((void **)&d_tail, 2 * 8));
    CK(cudaMalloc((void **)&d_table, 4 * sizeof(hq_kv_append_row)));
    CK(cudaMalloc((void **)&d_stats, sizeof(hq_stats)));
    CK(cudaMalloc(&d_ws, ws_bytes));
    cudaStream_t s;
    CK(cudaStreamCreate(&s));
    CK(cudaMemcpyAsync(d_kv, h_kv, n * 2, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(d_q, h_q, 128 * 128 * 4, cudaMemcpyHostToDevice, s));

    hq_params p;
    memset(&p, 0, sizeof p);
    p.tile = 128;
    p.lattice = HQ_E8;
    p.alpha = 1.0f;
    p.rice_k = atoi(argv[7]);
    p.rice_dk_last = atoi(argv[8]);
    p.seed = strtoull(argv[9], NULL, 10);
    p.dither = 1;
    p.chunk_tiles = 32;
    p.rotation = d_q;
    hq_kv_cache cache;
    HQ(hq_kv_init(&cache, heads, 128, &p, d_words, cap, d_offsets, max_chunks + 1, d_table, 4, d_tail, d_stats, s));
    const int64_t ld_head = tokens * 128;
    HQ(hq_kv_append(&cache, d_kv, t1, 128, ld_head, alpha, d_ws, ws_bytes, s));
    HQ(hq_kv_append(&cache, (const uint16_t *)d_kv + t1 * 128, t2, 128, ld_head, alpha, d_ws, ws_bytes, s));
    HQ(hq_kv_read(&cache, d_out, 1, tokens, 128, ld_head, s));
    HQ(hq_haar_rotation(p.seed, d_qdraw, s));

    hq_stats st;
    uint64_t *h_off = malloc((cache.chunks + 1) * 8);
    float *h_out = malloc(n * 4);
    if (!h_off || !h_out) return 5;
    CK(cudaMemcpyAsync(&st, d_stats, sizeof st, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_off, d_offsets, (cache.chunks + 1) * 8, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_out, d_out, n * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_q, d_qdraw, 128 * 128 * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    if (st.status != 0) {
        fprintf(stderr, "cache status %u (%s)\n", st.status, hq_status_string((int)st.status));
        return 6;
    }
    const uint64_t words = h_off[cache.chunks];
    uint32_t *h_words = malloc(words * 4 + 4);
    if (!h_words) return 5;
    CK(cudaMemcpy(h_words, d_words, words * 4, cudaMemcpyDeviceToHost));
    if (write_file(prefix, "stream.bin", h_words, words * 4) ||
        write_file(prefix, "offsets.bin", h_off, (cache.chunks + 1) * 8) ||
        write_file(prefix, "out.bin", h_out, n * 4) || write_file(prefix, "qdraw.bin", h_q, 128 * 128 * 4))
        return 9;
    printf("{\"payload_bits\": %llu, \"stream_words\": %llu, \"chunks\": %llu, \"appends\": %llu}\n",
           (unsigned long long)st.payload_bits, (unsigned long long)words, (unsigned long long)cache.chunks,
           (unsigned long long)cache.appends);
    cudaFree(d_kv);
    cudaFree(d_q);
    cudaFree(d_qdraw);
    cudaFree(d_out);
    cudaFree(d_words);
    cudaFree(d_offsets);
    cudaFree(d_tail);
    cudaFree(d_table);
    cudaFree(d_stats);
    cudaFree(d_ws);
    cudaStreamDestroy(s);
    free(h_kv);
    free(h_q);
    free(h_off);
    free(h_out);
    free(h_words);
    return 0;
}
