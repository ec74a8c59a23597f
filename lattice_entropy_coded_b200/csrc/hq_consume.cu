// hq_consume.cu -- decode fused into its consumer: the decoded tile feeds a dot
// product in registers instead of being written to HBM, so a weight matrix is
// read at its compressed size (about R/8 bytes per element) instead of 2 bytes
// of bf16.  Two consumers: a GEMV y = W x over a compressed matrix (one partial
// per 128-element tile, then row sums in column order, so the result does not
// depend on scheduling), and attention scores q . k over a compressed K cache.
// The decode itself is hq_decode.cuh's; the tile a dot product sees is exactly
// the bf16 tile hq_dequantize / hq_kv_read would store.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_decode.cuh"

namespace hq {

namespace {

// y[r] = sum of row r's tile partials, in tile-column order (one thread per row).
__global__ void __launch_bounds__(256) gemv_row_sums(const float *__restrict__ part, int64_t rows, int tpr,
                                                     float *__restrict__ y) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += stride) {
        const float *p = part + r * tpr;
        float acc = 0.0f;
        for (int t = 0; t < tpr; t++) acc = __fadd_rn(acc, p[t]);
        y[r] = acc;
    }
}

template <int LAT, bool DITHER, bool KV, int MODE>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(a.tcols * kSignWords + kWarpsPerCta * 2 * (kStageWords + kStagePad) +
                                 kWarpsPerCta * 128) *
                        sizeof(uint32_t);
    const bool small = a.k <= 4, mixed = a.k_last != a.k;
    auto kern = mixed ? decode_kernel<LAT, DITHER, KV, false, MODE, false, true>
                : small ? decode_kernel<LAT, DITHER, KV, true, MODE> : decode_kernel<LAT, DITHER, KV, false, MODE>;
    static LaunchPlan plans[3];
    unsigned grid = 0;
    // at most one CTA per round (the kernel deals rounds to CTAs first)
    cudaError_t e = plans[mixed ? 2 : small ? 1 : 0].grid(kern, kWarpsPerCta * 32, smem,
                                                           (unsigned long long)kRoundsPerChunk * a.n_chunks, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool KV, int MODE>
cudaError_t dispatch(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_t<HQ_Z, false, KV, MODE>(a, s);
    case HQ_Z * 2 + 1: return launch_t<HQ_Z, true, KV, MODE>(a, s);
    case HQ_A2 * 2: return launch_t<HQ_A2, false, KV, MODE>(a, s);
    case HQ_A2 * 2 + 1: return launch_t<HQ_A2, true, KV, MODE>(a, s);
    case HQ_D4 * 2: return launch_t<HQ_D4, false, KV, MODE>(a, s);
    case HQ_D4 * 2 + 1: return launch_t<HQ_D4, true, KV, MODE>(a, s);
    case HQ_E8 * 2: return launch_t<HQ_E8, false, KV, MODE>(a, s);
    case HQ_E8 * 2 + 1: return launch_t<HQ_E8, true, KV, MODE>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemv(int lattice, int dither, const DecodeArgs &a, float *y, cudaStream_t s) {
    cudaError_t e = dispatch<false, kGemvPartials>(lattice, dither, a, s);
    if (e != cudaSuccess) return e;
    const int64_t rows = a.map.rows;
    int64_t blocks = (rows + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    gemv_row_sums<<<(unsigned)blocks, 256, 0, s>>>(a.res, rows, a.tcols, y);
    return cudaGetLastError();
}

cudaError_t launch_kv_scores(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    if (a.rot) return launch_kv_scores_rot(lattice, dither, a, s);
    return dispatch<true, kKvScores>(lattice, dither, a, s);
}

}  // namespace hq
