// hq_encode.cu -- launchers of the quantize + encode kernels and of the rate pass
// with the sign diagonal and H_128 (the weights path and the default KV path).
// The kernels are in hq_encode.cuh.
#include "hq_encode.cuh"

namespace hq {

namespace {

template <int LAT, bool DITHER>
cudaError_t launch_tiny_t(const EncodeArgs &a, cudaStream_t s, bool small, bool mixed) {
    const size_t smem = (size_t)(a.tcols * kSignWords + kTinyMaxChunks * kStageWords) * sizeof(uint32_t) +
                        kTinyMaxChunks * (sizeof(TinyChunk) + sizeof(unsigned long long));
    auto kern = mixed ? encode_kernel_tiny<LAT, DITHER, false, false, true>
                : small ? encode_kernel_tiny<LAT, DITHER, true, false, false>
                        : encode_kernel_tiny<LAT, DITHER, false, false, false>;
    static LaunchPlan plans[3];
    unsigned grid = 0;
    cudaError_t e = plans[mixed ? 2 : small ? 1 : 0].grid(kern, kTinyWarps * 32, smem, 1, grid);
    if (e != cudaSuccess) return e;
    kern<<<1, kTinyWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

// One-token KV appends: every chunk is one tile.
template <int LAT, bool DITHER>
cudaError_t launch_tok_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(a.tcols * kSignWords + kTinyMaxChunks * kTokStageWords) * sizeof(uint32_t) +
                        kTinyMaxChunks * (sizeof(TinyChunk) + sizeof(unsigned long long));
    auto kern = encode_kernel_tok<LAT, DITHER, false>;
    static LaunchPlan plan;
    unsigned grid = 0;
    cudaError_t e = plan.grid(kern, kTinyWarps * 32, smem, 1, grid);
    if (e != cudaSuccess) return e;
    kern<<<1, kTinyWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int LAT, bool DITHER>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
    const bool small = a.k <= 4;
    const bool mixed = a.k_last != a.k;   // a second Rice parameter: per-warp or grouped forms only
    cudaError_t e;
    unsigned grid = 0;
    // by size: one CTA for the whole launch up to kTinyMaxChunks chunks; the wide form
    // while every chunk gets a 16-warp group of its own in one wave (2 CTAs per SM); the
    // grouped form up to three quarters of the per-warp form's resident warps (2 CTAs of
    // kWarpsPerCta per SM), or all of them with dither, because a warp encoding a lone
    // chunk is latency-bound and four warps per chunk finish it sooner (B200, E8 4 bps:
    // 1200 chunks 45.5 -> 37.9 us, 69.5 -> 48.2 us with dither); else the per-warp form
    int mode = g_encode_path;
    if (mode == 0) {
        int dev = 0, sms = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        const unsigned long long per_warp = 2ull * kWarpsPerCta * (unsigned long long)sms;
        mode = (a.n_chunks <= (unsigned long long)kTinyMaxChunks) ? 4
               : (a.n_chunks <= 2ull * (unsigned long long)sms) ? 3
               : (a.n_chunks <= (DITHER ? per_warp : per_warp * 3 / 4)) ? 2 : 1;
    }
    if (mode == 4 && a.n_chunks > (unsigned long long)kTinyMaxChunks) mode = 1;
    if (mixed && mode == 3) mode = 2;
    const bool batched = a.batch > 1;
    if (batched) mode = 1;   // a strided batch runs the per-warp form, which keeps per-item state
    if (mode == 4) {
        // a one-token KV append (one tile per chunk) with a single Rice parameter
        if (a.map.kv && a.map.tokens == 1 && !mixed) return launch_tok_t<LAT, DITHER>(a, s);
        return launch_tiny_t<LAT, DITHER>(a, s, small, mixed);
    }
    // the multi-CTA forms share the workspace: look-back words, ticket, done counter and
    // stats accumulator, cleared by one memset
    if ((e = cudaMemsetAsync(a.lookback, 0, encode_scratch_bytes(a.n_chunks, batched ? a.batch : 1), s)) !=
        cudaSuccess)
        return e;
    if (mode == 3) {
        const size_t smem =
            (size_t)(a.tcols * kSignWords + 2 * kStageWords) * sizeof(uint32_t) + sizeof(WideCtl);
        auto kern = encode_kernel_wide<LAT, DITHER>;
        static LaunchPlan plan;
        if ((e = plan.grid(kern, kWideWarps * 32, smem, a.n_chunks, grid)) != cudaSuccess) return e;
        kern<<<grid, kWideWarps * 32, smem, s>>>(a);
    } else if (mode == 2) {
        const size_t smem = (size_t)(a.tcols * kSignWords + kGroups * 2 * kStageWords +
                                     kWarpsPerCta * 32 * kGroupSlotWords) * sizeof(uint32_t) +
                            kGroups * sizeof(GroupCtl);
        auto kern = mixed ? encode_kernel_grouped<LAT, DITHER, false, false, true>
                    : small ? encode_kernel_grouped<LAT, DITHER, true, false> : encode_kernel_grouped<LAT, DITHER, false, false>;
        static LaunchPlan plans[3];
        if ((e = plans[mixed ? 2 : small ? 1 : 0].grid(kern, kWarpsPerCta * 32, smem, (a.n_chunks + kGroups - 1) / kGroups,
                                                        grid)) != cudaSuccess)
            return e;
        kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    } else {
        const size_t smem =
            (size_t)(a.tcols * kSignWords + kWarpsPerCta * 2 * kStageWords + kWarpsPerCta * 32 * kInSlotWords) *
            sizeof(uint32_t);
        // weights whose rows hold whole rounds (cols a multiple of 8 tiles): every round is one
        // 2 KB run of x, 16-byte aligned (x, ld and the item stride are checked at the API),
        // brought in by one bulk copy.  Fewer than 2^27 chunks (more than device memory holds)
        // keep that kernel's chunk arithmetic 32-bit.
        const bool bulk = !mixed && !a.map.kv && a.map.cols % (kTilesPerRound * kTile) == 0 &&
                          a.n_chunks < (1ull << 27) &&
                          ((uintptr_t)a.x & 15u) == 0 && a.map.ld % 8 == 0 && (a.batch <= 1 || a.item_x_stride % 8 == 0);
        auto kern = mixed ? encode_kernel<LAT, DITHER, false, true>
                    : bulk ? (small ? encode_kernel<LAT, DITHER, true, false, true>
                                    : encode_kernel<LAT, DITHER, false, false, true>)
                    : small ? encode_kernel<LAT, DITHER, true> : encode_kernel<LAT, DITHER, false>;
        int plan_i = mixed ? 2 : (small ? 1 : 0) + (bulk ? 3 : 0);
        if constexpr (LAT == HQ_E8) {
            // E8 weights at the common rates (k = 1 .. 4): the Rice parameter compiled in
            if (bulk && a.k >= 1 && a.k <= 4) {
                plan_i = 4 + a.k;
                kern = a.k == 1   ? encode_kernel<LAT, DITHER, true, false, true, 1>
                       : a.k == 2 ? encode_kernel<LAT, DITHER, true, false, true, 2>
                       : a.k == 3 ? encode_kernel<LAT, DITHER, true, false, true, 3>
                                  : encode_kernel<LAT, DITHER, true, false, true, 4>;
            }
        }
        if (a.map.kv && !mixed) {
            // a KV append (a prefill, or many tokens): the weights tile map compiled out, and for
            // E8 with dither at k = 0 (the KV caches' rates near 2 bits) the Rice parameter too
            plan_i = 9 + (small ? 1 : 0);
            kern = small ? encode_kernel<LAT, DITHER, true, false, false, -1, true>
                         : encode_kernel<LAT, DITHER, false, false, false, -1, true>;
            if constexpr (LAT == HQ_E8 && DITHER) {
                if (a.k == 0) {
                    plan_i = 11;
                    kern = encode_kernel<LAT, DITHER, true, false, false, 0, true>;
                }
            }
        }
        static LaunchPlan plans[12];
        if ((e = plans[plan_i].grid(kern, kWarpsPerCta * 32, smem, (a.n_chunks + kWarpsPerCta - 1) / kWarpsPerCta,
                                    grid)) != cudaSuccess)
            return e;
        kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    }
    return cudaGetLastError();
}

template <int LAT, bool DITHER>
cudaError_t launch_rate_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)a.tcols * kSignWords * sizeof(uint32_t);
    auto kern = rate_kernel<LAT, DITHER, false>;
    static LaunchPlan plan;
    unsigned grid = 0;
    cudaError_t e = plan.grid(kern, kWarpsPerCta * 32, smem, (a.n_chunks + kWarpsPerCta - 1) / kWarpsPerCta, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarpsPerCta * 32, smem, s>>>(a);
    return cudaGetLastError();
}


}  // namespace

cudaError_t launch_encode(int lattice, int dither, const EncodeArgs &a, cudaStream_t s) {
    if (a.rot) return launch_encode_rot(lattice, dither, a, s);
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_t<HQ_Z, false>(a, s);
    case HQ_Z * 2 + 1: return launch_t<HQ_Z, true>(a, s);
    case HQ_A2 * 2: return launch_t<HQ_A2, false>(a, s);
    case HQ_A2 * 2 + 1: return launch_t<HQ_A2, true>(a, s);
    case HQ_D4 * 2: return launch_t<HQ_D4, false>(a, s);
    case HQ_D4 * 2 + 1: return launch_t<HQ_D4, true>(a, s);
    case HQ_E8 * 2: return launch_t<HQ_E8, false>(a, s);
    case HQ_E8 * 2 + 1: return launch_t<HQ_E8, true>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_rate(int lattice, int dither, const EncodeArgs &a, cudaStream_t s) {
    if (a.rot) return launch_rate_rot(lattice, dither, a, s);
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_rate_t<HQ_Z, false>(a, s);
    case HQ_Z * 2 + 1: return launch_rate_t<HQ_Z, true>(a, s);
    case HQ_A2 * 2: return launch_rate_t<HQ_A2, false>(a, s);
    case HQ_A2 * 2 + 1: return launch_rate_t<HQ_A2, true>(a, s);
    case HQ_D4 * 2: return launch_rate_t<HQ_D4, false>(a, s);
    case HQ_D4 * 2 + 1: return launch_rate_t<HQ_D4, true>(a, s);
    case HQ_E8 * 2: return launch_rate_t<HQ_E8, false>(a, s);
    case HQ_E8 * 2 + 1: return launch_rate_t<HQ_E8, true>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hq

