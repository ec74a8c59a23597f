// hq_rot_encode.cu -- launchers of the quantize + encode kernel and of the rate pass
// with the dense KV rotation (a 128 x 128 orthogonal matrix per cache in place of
// the sign diagonal and H_128; explainer pages, "Methodology" 4).  The kernels are
// the grouped, single-CTA and one-token forms and the rate kernel of hq_encode.cuh
// with ROT = true, instantiated in this file of their own so that they compile in
// parallel with the rest.
#include "hq_encode.cuh"

namespace hq {

namespace {

// Up to kTinyMaxChunksRot chunks: one CTA for the whole launch.  Beyond: the grouped
// form, four warps per chunk, one CTA of kRotGroups groups per SM (the rotation's shared
// form and per-warp buffers, 194 KB).
// A one-token append (one tile per chunk) with a single Rice parameter: the one-token
// form, a half-warp per chunk, up to kTinyMaxChunks chunks.
template <int LAT, bool DITHER>
cudaError_t launch_rot_t(const EncodeArgs &a, cudaStream_t s) {
    const bool small = a.k <= 4, mixed = a.k_last != a.k;
    const bool single_cta = g_encode_path == 0 || g_encode_path == 4;
    if (single_cta && a.map.kv && a.map.tokens == 1 && !mixed && a.n_chunks <= (unsigned long long)kTinyMaxChunks) {
        const size_t smem = rot_smem_bytes(kTinyWarps) +
                            (size_t)(a.tcols * kSignWords + kTinyMaxChunks * kTokStageWords) * sizeof(uint32_t) +
                            kTinyMaxChunks * (sizeof(TinyChunk) + sizeof(unsigned long long));
        auto kern = encode_kernel_tok<LAT, DITHER, true>;
        static LaunchPlan kplan;
        unsigned kgrid = 0;
        cudaError_t e = kplan.grid(kern, kTinyWarps * 32, smem, 1, kgrid);
        if (e != cudaSuccess) return e;
        kern<<<1, kTinyWarps * 32, smem, s>>>(a);
        return cudaGetLastError();
    }
    if (a.n_chunks <= (unsigned long long)kTinyMaxChunksRot && single_cta) {
        const size_t smem = kRotSmemBytes + (size_t)(a.tcols * kSignWords + kTinyMaxChunksRot * kStageWords) *
                                                sizeof(uint32_t) +
                            kTinyMaxChunksRot * (sizeof(TinyChunk) + sizeof(unsigned long long));
        auto kern = mixed ? encode_kernel_tiny<LAT, DITHER, false, true, true>
                    : small ? encode_kernel_tiny<LAT, DITHER, true, true, false>
                            : encode_kernel_tiny<LAT, DITHER, false, true, false>;
        static LaunchPlan tplans[3];
        unsigned tgrid = 0;
        cudaError_t e = tplans[mixed ? 2 : small ? 1 : 0].grid(kern, kTinyWarps * 32, smem, 1, tgrid);
        if (e != cudaSuccess) return e;
        kern<<<1, kTinyWarps * 32, smem, s>>>(a);
        return cudaGetLastError();
    }
    cudaError_t me = cudaMemsetAsync(a.lookback, 0, encode_scratch_bytes(a.n_chunks), s);
    if (me != cudaSuccess) return me;
    constexpr int W = kRotGroups * kGroupWarps;
    const size_t smem = rot_smem_bytes(W) +
                        (size_t)(a.tcols * kSignWords + kRotGroups * 2 * kStageWords + W * 32 * kGroupSlotWords) *
                            sizeof(uint32_t) +
                        kRotGroups * sizeof(GroupCtl);
    auto kern = mixed ? encode_kernel_grouped<LAT, DITHER, false, true, true>
                : small ? encode_kernel_grouped<LAT, DITHER, true, true> : encode_kernel_grouped<LAT, DITHER, false, true>;
    static LaunchPlan plans[3];
    unsigned grid = 0;
    // one CTA per chunk up to one per SM: a short append spreads over as many SMs as it
    // has chunks (the rotation is bound by each SM's fma rate), idle groups exit at once
    cudaError_t e = plans[mixed ? 2 : small ? 1 : 0].grid(kern, W * 32, smem, a.n_chunks, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, W * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int LAT, bool DITHER>
cudaError_t launch_rate_rot_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem = kRotSmemBytes + (size_t)a.tcols * kSignWords * sizeof(uint32_t);
    auto kern = rate_kernel<LAT, DITHER, true>;
    static LaunchPlan plan;
    unsigned grid = 0;
    cudaError_t e = plan.grid(kern, kWarpsPerCta * 32, smem, (a.n_chunks + kWarpsPerCta - 1) / kWarpsPerCta, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode_rot(int lattice, int dither, const EncodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_rot_t<HQ_Z, false>(a, s);
    case HQ_Z * 2 + 1: return launch_rot_t<HQ_Z, true>(a, s);
    case HQ_A2 * 2: return launch_rot_t<HQ_A2, false>(a, s);
    case HQ_A2 * 2 + 1: return launch_rot_t<HQ_A2, true>(a, s);
    case HQ_D4 * 2: return launch_rot_t<HQ_D4, false>(a, s);
    case HQ_D4 * 2 + 1: return launch_rot_t<HQ_D4, true>(a, s);
    case HQ_E8 * 2: return launch_rot_t<HQ_E8, false>(a, s);
    case HQ_E8 * 2 + 1: return launch_rot_t<HQ_E8, true>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_rate_rot(int lattice, int dither, const EncodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_rate_rot_t<HQ_Z, false>(a, s);
    case HQ_Z * 2 + 1: return launch_rate_rot_t<HQ_Z, true>(a, s);
    case HQ_A2 * 2: return launch_rate_rot_t<HQ_A2, false>(a, s);
    case HQ_A2 * 2 + 1: return launch_rate_rot_t<HQ_A2, true>(a, s);
    case HQ_D4 * 2: return launch_rate_rot_t<HQ_D4, false>(a, s);
    case HQ_D4 * 2 + 1: return launch_rate_rot_t<HQ_D4, true>(a, s);
    case HQ_E8 * 2: return launch_rate_rot_t<HQ_E8, false>(a, s);
    case HQ_E8 * 2 + 1: return launch_rate_rot_t<HQ_E8, true>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hq
