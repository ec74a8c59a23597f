// hq_shard.cu -- hq_offsets_add: move a stream's chunk offsets by a base word index.
//
// A set of tensors is coded across GPUs as independent shards: each GPU writes its own
// streams and offsets, with no exchange on the coding path (chunks depend on one another
// only through the exclusive scan of their sizes, which stays inside one call).  Where
// the shards are to read as one global stream, each GPU learns the global word index at
// which its part starts (one gather of the per-GPU word counts) and moves its offsets by
// it with this kernel.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_internal.h"

namespace hq {
namespace {

__global__ void offsets_add_kernel(unsigned long long *off, unsigned long long n, unsigned long long base) {
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    for (unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        off[i] += base;
}

}  // namespace
}  // namespace hq

extern "C" {

int hq_offsets_add(uint64_t *d_offsets, uint64_t count, uint64_t base, void *cuda_stream) {
    if (count == 0) return HQ_OK;
    if (!d_offsets || ((uintptr_t)d_offsets % 8) != 0) return HQ_EINVAL;
    const unsigned threads = 256;
    unsigned long long blocks = (count + threads - 1) / threads;
    if (blocks > 148ull * 8ull) blocks = 148ull * 8ull;   // grid-stride beyond a few waves
    hq::offsets_add_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)cuda_stream>>>(
        (unsigned long long *)d_offsets, (unsigned long long)count, (unsigned long long)base);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ECUDA;
}

}  // extern "C"
