/* A C program that uses libhq.so through include/hq.h alone (plus the CUDA
 * runtime for device memory): quantize a bf16 matrix read from a file, check
 * hq_rate against hq_quantize's stats, dequantize it to bf16, run the fused GEMV,
 * and write the stream, offsets, reconstruction and GEMV result to files for the
 * test that drives it to compare with the oracle.
 *
 *   hq_roundtrip IN.bin ROWS COLS LATTICE ALPHA K SEED OUTPREFIX
 *
 * IN.bin holds ROWS*COLS bf16 values (uint16, row-major) followed by COLS bf16
 * values of the GEMV vector.  Exit status 0 on success; messages on stderr. */
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

static int write_file(const char *prefix, const char *name, const void *p, size_t n) {
    char path[1024];
    snprintf(path, sizeof path, "%s%s", prefix, name);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(p, 1, n, f) != n) return 1;
    return fclose(f) != 0;
}

int main(int argc, char **argv) {
    if (argc != 9) {
        fprintf(stderr, "usage: %s IN.bin ROWS COLS LATTICE ALPHA K SEED OUTPREFIX\n", argv[0]);
        return 1;
    }
    const int64_t rows = atoll(argv[2]), cols = atoll(argv[3]);
    hq_params p;
    memset(&p, 0, sizeof p);
    p.tile = 128;
    p.lattice = atoi(argv[4]);
    p.alpha = (float)atof(argv[5]);
    p.rice_k = atoi(argv[6]);
    p.seed = strtoull(argv[7], NULL, 10);
    p.dither = 0;
    p.chunk_tiles = 32;
    const char *prefix = argv[8];
    if (hq_device_check() != HQ_OK) {
        fprintf(stderr, "no sm_100 device\n");
        return 4;
    }

    const size_t n = (size_t)rows * (size_t)cols;
    uint16_t *h_in = malloc((n + (size_t)cols) * 2);
    FILE *f = fopen(argv[1], "rb");
    if (!h_in || !f || fread(h_in, 2, n + (size_t)cols, f) != n + (size_t)cols) return 5;
    fclose(f);

    uint64_t cap = 0, nch = 0;
    HQ(hq_stream_bound(rows, cols, &p, 0, &cap, &nch));
    size_t ws_bytes = 0, gemv_ws = 0;
    HQ(hq_workspace_bytes(nch, &ws_bytes));
    HQ(hq_gemv_workspace_bytes(rows, cols, &gemv_ws));

    void *d_x, *d_ws, *d_out, *d_v, *d_gws;
    uint32_t *d_stream;
    uint64_t *d_off;
    hq_stats *d_stats, *d_rate;
    float *d_y;
    CK(cudaMalloc(&d_x, n * 2));
    CK(cudaMalloc(&d_v, (size_t)cols * 2));
    CK(cudaMalloc((void **)&d_stream, cap * 4));
    CK(cudaMalloc((void **)&d_off, (nch + 1) * 8));
    CK(cudaMalloc((void **)&d_stats, sizeof(hq_stats)));
    CK(cudaMalloc((void **)&d_rate, sizeof(hq_stats)));
    CK(cudaMalloc(&d_ws, ws_bytes));
    CK(cudaMalloc(&d_out, n * 2));
    CK(cudaMalloc(&d_gws, gemv_ws));
    CK(cudaMalloc((void **)&d_y, (size_t)rows * 4));
    cudaStream_t s;
    CK(cudaStreamCreate(&s));
    CK(cudaMemcpyAsync(d_x, h_in, n * 2, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(d_v, h_in + n, (size_t)cols * 2, cudaMemcpyHostToDevice, s));

    HQ(hq_quantize(d_x, rows, cols, cols, &p, d_stream, cap, d_off, d_stats, d_ws, ws_bytes, s));
    HQ(hq_rate(d_x, rows, cols, cols, &p, d_rate, s));
    hq_stats st, rt;
    CK(cudaMemcpyAsync(&st, d_stats, sizeof st, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(&rt, d_rate, sizeof rt, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    if (st.status != 0 || st.stream_words > cap) {
        fprintf(stderr, "quantize status %u (%s)\n", st.status, hq_status_string((int)st.status));
        return 6;
    }
    if (rt.payload_bits != st.payload_bits || rt.stream_words != st.stream_words || rt.max_symbol != st.max_symbol) {
        fprintf(stderr, "hq_rate disagrees with hq_quantize\n");
        return 7;
    }
    HQ(hq_dequantize(d_stream, st.stream_words, d_off, rows, cols, &p, d_out, 0, cols, d_stats, s));
    HQ(hq_gemv(d_stream, st.stream_words, d_off, rows, cols, &p, d_v, d_y, d_gws, gemv_ws, NULL, s));

    uint32_t *h_stream = malloc(st.stream_words * 4 + 4);
    uint64_t *h_off = malloc((nch + 1) * 8);
    uint16_t *h_out = malloc(n * 2);
    float *h_y = malloc((size_t)rows * 4);
    if (!h_stream || !h_off || !h_out || !h_y) return 5;
    CK(cudaMemcpyAsync(h_stream, d_stream, st.stream_words * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_off, d_off, (nch + 1) * 8, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_out, d_out, n * 2, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(h_y, d_y, (size_t)rows * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(&st, d_stats, sizeof st, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    if (st.status != 0) {
        fprintf(stderr, "dequantize status %u\n", st.status);
        return 8;
    }
    if (write_file(prefix, "stream.bin", h_stream, rt.stream_words * 4) ||
        write_file(prefix, "offsets.bin", h_off, (nch + 1) * 8) || write_file(prefix, "out.bin", h_out, n * 2) ||
        write_file(prefix, "y.bin", h_y, (size_t)rows * 4))
        return 9;
    printf("{\"payload_bits\": %llu, \"stream_words\": %llu, \"chunks\": %llu}\n",
           (unsigned long long)rt.payload_bits, (unsigned long long)rt.stream_words, (unsigned long long)nch);
    cudaFree(d_x);
    cudaFree(d_v);
    cudaFree(d_stream);
    cudaFree(d_off);
    cudaFree(d_stats);
    cudaFree(d_rate);
    cudaFree(d_ws);
    cudaFree(d_out);
    cudaFree(d_gws);
    cudaFree(d_y);
    cudaStreamDestroy(s);
    free(h_in);
    free(h_stream);
    free(h_off);
    free(h_out);
    free(h_y);
    return 0;
}
