// hq_decode.cu -- decode + dequantize kernel (HyperQuant "Methodology" sections
// 1-4 inverted): Rice planes -> symbols -> re-inserted membership bits ->
// lattice point [- dither] -> scale -> FWHT-128 -> sign -> bf16 (or fp32).
// This file instantiates and launches the stored-tile form; the kernel itself is
// in hq_decode.cuh.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_decode.cuh"

namespace hq {

namespace {

template <int LAT, bool DITHER, bool KV>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(a.tcols * kSignWords + kWarpsPerCta * 2 * (kStageWords + kStagePad) +
                                 kWarpsPerCta * 128) *
                        sizeof(uint32_t);
    const bool small = a.k <= 4, mixed = a.k_last != a.k;
    auto kern = mixed ? decode_kernel<LAT, DITHER, KV, false, kStoreTiles, false, true>
                : small ? decode_kernel<LAT, DITHER, KV, true, kStoreTiles> : decode_kernel<LAT, DITHER, KV, false, kStoreTiles>;
    int plan_i = mixed ? 2 : small ? 1 : 0;
    if constexpr (LAT == HQ_E8 && !KV) {
        // E8 weights at the common rates (k = 1 .. 4): the Rice parameter compiled in
        // (to bf16, the fp32 store compiled out)
        if (!mixed && !a.out_fp32 && a.k >= 1 && a.k <= 4) {
            plan_i = 2 + a.k;
            kern = a.k == 1   ? decode_kernel<LAT, DITHER, KV, true, kStoreBf16, false, false, 1>
                   : a.k == 2 ? decode_kernel<LAT, DITHER, KV, true, kStoreBf16, false, false, 2>
                   : a.k == 3 ? decode_kernel<LAT, DITHER, KV, true, kStoreBf16, false, false, 3>
                              : decode_kernel<LAT, DITHER, KV, true, kStoreBf16, false, false, 4>;
        }
    }
    if constexpr (LAT == HQ_E8 && DITHER && KV) {
        // a KV cache read to bf16 at k = 0 (the KV caches' rates near 2 bits): k compiled in
        if (!mixed && !a.out_fp32 && a.k == 0) {
            plan_i = 7;
            kern = decode_kernel<LAT, DITHER, KV, true, kStoreBf16, false, false, 0>;
        }
    }
    static LaunchPlan plans[8];
    unsigned grid = 0;
    // at most one CTA per round (the kernel deals rounds to CTAs first)
    cudaError_t e = plans[plan_i].grid(kern, kWarpsPerCta * 32, smem, (unsigned long long)kRoundsPerChunk * a.n_chunks,
                                       grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool KV>
cudaError_t dispatch(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_t<HQ_Z, false, KV>(a, s);
    case HQ_Z * 2 + 1: return launch_t<HQ_Z, true, KV>(a, s);
    case HQ_A2 * 2: return launch_t<HQ_A2, false, KV>(a, s);
    case HQ_A2 * 2 + 1: return launch_t<HQ_A2, true, KV>(a, s);
    case HQ_D4 * 2: return launch_t<HQ_D4, false, KV>(a, s);
    case HQ_D4 * 2 + 1: return launch_t<HQ_D4, true, KV>(a, s);
    case HQ_E8 * 2: return launch_t<HQ_E8, false, KV>(a, s);
    case HQ_E8 * 2 + 1: return launch_t<HQ_E8, true, KV>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    if (a.rot) return launch_decode_rot(lattice, dither, a, s);
    return a.map.kv ? dispatch<true>(lattice, dither, a, s) : dispatch<false>(lattice, dither, a, s);
}

}  // namespace hq
