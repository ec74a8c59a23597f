// hq_debug.cu -- hq_debug_nearest: the device nearest-point decoders of the four
// lattices (the ones the encode and decode kernels inline) run on caller-given
// vectors, so tests can compare them with the oracle on inputs the transform
// would rarely produce (points on Voronoi-cell boundaries, exact ties, large
// magnitudes).  Method: HyperQuant explainer pages, "Methodology" section 2.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_device.cuh"

namespace hq {
namespace {

template <int LAT>
__global__ void __launch_bounds__(256) nearest_kernel(const float *__restrict__ v, int64_t n, int32_t *__restrict__ q) {
    constexpr int N = Lattice<LAT>::N;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n; b += stride) {
        float x[N];
        int32_t c[N];
#pragma unroll
        for (int i = 0; i < N; i++) x[i] = v[b * N + i];
        Lattice<LAT>::nearest(x, c);
#pragma unroll
        for (int i = 0; i < N; i++) q[b * N + i] = c[i];
    }
}

template <int LAT>
cudaError_t launch_nearest(const float *v, int64_t n, int32_t *q, cudaStream_t s) {
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    nearest_kernel<LAT><<<(unsigned)blocks, 256, 0, s>>>(v, n, q);
    return cudaGetLastError();
}

}  // namespace
}  // namespace hq

extern "C" int hq_debug_nearest(int lattice, const float *d_v, int64_t n_blocks, int32_t *d_q, void *cuda_stream) {
    using namespace hq;
    if (lattice < HQ_Z || lattice > HQ_E8 || n_blocks < 0) return HQ_EINVAL;
    if (n_blocks == 0) return HQ_OK;
    if (!d_v || !d_q || ((uintptr_t)d_v & 3u) || ((uintptr_t)d_q & 3u)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    cudaError_t e = cudaErrorInvalidValue;
    switch (lattice) {
    case HQ_Z: e = launch_nearest<HQ_Z>(d_v, n_blocks, d_q, s); break;
    case HQ_A2: e = launch_nearest<HQ_A2>(d_v, n_blocks, d_q, s); break;
    case HQ_D4: e = launch_nearest<HQ_D4>(d_v, n_blocks, d_q, s); break;
    case HQ_E8: e = launch_nearest<HQ_E8>(d_v, n_blocks, d_q, s); break;
    }
    return e == cudaSuccess ? HQ_OK : HQ_ECUDA;
}
