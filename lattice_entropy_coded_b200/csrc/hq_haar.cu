// hq_haar.cu -- draws the dense KV rotation: a Haar-uniform 128 x 128 orthogonal
// matrix per seed (explainer pages, "Methodology" 4: each layer's keys and values
// are rotated by a full Haar-uniform matrix or by the cheap sign diagonal).
//
// G[i][j] is the standard normal draw e = 128 i + j: h = splitmix64(seed ^ "ROTN",
// e), u1 = (hi32(h) + 1/2) 2^-32, u2 = lo32(h) 2^-32, g = sqrt(-2 ln u1) cos(2 pi u2)
// (Box-Muller, cosine branch, double).  Q is the orthogonal factor of G = Q R with a
// positive diagonal in R; that factor is unique and Haar-distributed (Mezzadri,
// "How to generate random matrices from the classical compact groups", 2007).  It is
// computed here by modified Gram-Schmidt in double (norms are positive, so the
// diagonal of R is too) and rounded once to fp32.  Any QR method gives the same
// factor up to rounding: against a Householder QR the double results differ by about
// cond(G) x 2^-53, far below the fp32 rounding, so the fp32 matrices agree to within
// one unit in the last place.
//
// One CTA, the matrix in shared memory (132 KB of doubles, column-major so that a
// warp walks a column with consecutive lanes); 128 sequential steps.  Runs once per
// cache, not on the append or read path.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_device.cuh"

namespace hq {

namespace {

constexpr int kHaarThreads = 512;
constexpr int kHaarPitch = 129;   // doubles per column: consecutive columns start in different banks
constexpr uint64_t kRotSalt = 0x524F544Eull;   // "ROTN"
constexpr size_t kHaarSmemBytes = (size_t)128 * kHaarPitch * sizeof(double) + 16;

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kHaarThreads, 1) haar_kernel(uint64_t seed, float *q) {
    extern __shared__ __align__(16) double A[];   // column j at A + j * kHaarPitch; then one double
    double *norm = A + 128 * kHaarPitch;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;

    for (int e = tid; e < 128 * 128; e += blockDim.x) {
        const uint64_t h = splitmix64(seed ^ kRotSalt, (uint64_t)e);
        const double u1 = ((double)(h >> 32) + 0.5) * 0x1p-32;
        const double u2 = (double)(h & 0xFFFFFFFFull) * 0x1p-32;
        A[(e & 127) * kHaarPitch + (e >> 7)] = sqrt(-2.0 * log(u1)) * cospi(2.0 * u2);
    }
    __syncthreads();

    for (int k = 0; k < 128; k++) {
        double *ak = A + k * kHaarPitch;
        if (warp == 0) {
            double s = 0.0;
            for (int i = lane; i < 128; i += 32) s = fma(ak[i], ak[i], s);
            s = warp_sum_f64(s);
            if (lane == 0) *norm = sqrt(s);
        }
        __syncthreads();
        const double nk = *norm;
        for (int i = tid; i < 128; i += blockDim.x) ak[i] = ak[i] / nk;
        __syncthreads();
        for (int j = k + 1 + warp; j < 128; j += nw) {
            double *aj = A + j * kHaarPitch;
            double r = 0.0;
            for (int i = lane; i < 128; i += 32) r = fma(ak[i], aj[i], r);
            r = warp_sum_f64(r);
            for (int i = lane; i < 128; i += 32) aj[i] = fma(-r, ak[i], aj[i]);
        }
        __syncthreads();
    }

    for (int e = tid; e < 128 * 128; e += blockDim.x) q[e] = __double2float_rn(A[(e & 127) * kHaarPitch + (e >> 7)]);
}

}  // namespace

cudaError_t launch_haar(uint64_t seed, float *q, cudaStream_t s) {
    static LaunchPlan plan;   // sets the shared-memory attribute once per device
    unsigned grid = 0;
    cudaError_t e = plan.grid(haar_kernel, kHaarThreads, kHaarSmemBytes, 1, grid);
    if (e != cudaSuccess) return e;
    haar_kernel<<<1, kHaarThreads, kHaarSmemBytes, s>>>(seed, q);
    return cudaGetLastError();
}

}  // namespace hq
