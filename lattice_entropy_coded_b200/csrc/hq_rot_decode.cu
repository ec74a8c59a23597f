// hq_rot_decode.cu -- the decoder of a KV cache with the dense rotation (a 128 x 128
// orthogonal matrix in place of the sign diagonal and H_128; explainer pages,
// "Methodology" 4): hq_kv_read's stored tiles and hq_kv_scores' dot products.  The
// kernel is hq_decode.cuh's with ROT = true, instantiated here so that it compiles in
// parallel with the rest.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_decode.cuh"

namespace hq {

namespace {

// One CTA of kRotDecodeWarps warps per SM: the rotation's shared form of Q^T and the
// per-warp rotation buffers come on top of two stages per warp (223 KB at 12 warps).
template <int LAT, bool DITHER, int MODE>
cudaError_t launch_rot_t(const DecodeArgs &a, cudaStream_t s) {
    constexpr int W = kRotDecodeWarps;
    const size_t smem = rot_smem_bytes(W) + (size_t)(a.tcols * kSignWords + W * 2 * (kStageWords + kStagePad) + W * 128) *
                                                sizeof(uint32_t);
    const bool small = a.k <= 4, mixed = a.k_last != a.k;
    auto kern = mixed ? decode_kernel<LAT, DITHER, true, false, MODE, true, true>
                : small ? decode_kernel<LAT, DITHER, true, true, MODE, true> : decode_kernel<LAT, DITHER, true, false, MODE, true>;
    static LaunchPlan plans[3];
    unsigned grid = 0;
    // one CTA per round up to one per SM (the kernel deals rounds to CTAs first)
    cudaError_t e = plans[mixed ? 2 : small ? 1 : 0].grid(kern, W * 32, smem,
                                                           (unsigned long long)kRoundsPerChunk * a.n_chunks, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, W * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_rot_t<HQ_Z, false, MODE>(a, s);
    case HQ_Z * 2 + 1: return launch_rot_t<HQ_Z, true, MODE>(a, s);
    case HQ_A2 * 2: return launch_rot_t<HQ_A2, false, MODE>(a, s);
    case HQ_A2 * 2 + 1: return launch_rot_t<HQ_A2, true, MODE>(a, s);
    case HQ_D4 * 2: return launch_rot_t<HQ_D4, false, MODE>(a, s);
    case HQ_D4 * 2 + 1: return launch_rot_t<HQ_D4, true, MODE>(a, s);
    case HQ_E8 * 2: return launch_rot_t<HQ_E8, false, MODE>(a, s);
    case HQ_E8 * 2 + 1: return launch_rot_t<HQ_E8, true, MODE>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_rot(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    if (!a.map.kv) return cudaErrorInvalidValue;
    return dispatch<kStoreTiles>(lattice, dither, a, s);
}

cudaError_t launch_kv_scores_rot(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    if (!a.map.kv) return cudaErrorInvalidValue;
    return dispatch<kKvScores>(lattice, dither, a, s);
}

}  // namespace hq
