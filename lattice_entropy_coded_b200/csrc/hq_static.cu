// hq_static.cu -- hq_quantize_static: the weights-path quantize + encode for
// callers that cannot allocate device memory.  The encoder's scratch (the
// chunk look-back words, the chunk ticket and done counter, the stats
// accumulator) lives in a fixed array that is part of this library's device
// image instead of in a caller workspace.
//
// In host code the array's name is a host-side stand-in, not a device address:
// every call asks the runtime for the array's address in the current context
// (cudaGetSymbolAddress, with the caller's device current) and passes that to
// the kernels.  Asking on every call, rather than caching per device, keeps the
// address right after a cudaDeviceReset or in another context on the same device.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "hq_internal.h"

using namespace hq;

namespace {

constexpr size_t kStaticScratchBytes = HQ_STATIC_SCRATCH_BYTES;

// Look-back words (8 bytes per chunk), the ticket and done words, the stats accumulator.
static __device__ __align__(256) unsigned char g_hq_scratch[kStaticScratchBytes];

// Device address of the scratch in the current context.
int scratch_address(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_hq_scratch) != cudaSuccess || !p) return HQ_ECUDA;
    *out = p;
    return HQ_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" {

int hq_quantize_static(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, uint32_t *d_stream,
                       uint64_t cap_words, uint64_t *d_offsets, hq_stats *d_stats, void *cuda_stream) {
    // the same argument rules as hq_quantize, then the scratch limit
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    const uint64_t nch = chunks_of(rows, cols);
    if (nch > HQ_STATIC_MAX_CHUNKS) return HQ_EUNSUPPORTED;   // beyond the fixed scratch
    if (!d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (nch == 0) {
        if (d_stats && cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
        return cudaMemsetAsync(d_offsets, 0, sizeof(uint64_t), s) == cudaSuccess ? HQ_OK : HQ_ECUDA;
    }
    if (!x || !aligned(x, 16) || ld < cols || ld % 8) return HQ_EINVAL;
    if (!d_stream || !aligned(d_stream, 4)) return HQ_EINVAL;
    void *scratch = nullptr;
    if ((rc = scratch_address(&scratch))) return rc;
    // the previous call's look-back words, ticket, counter and stats are still in the
    // array: the launcher clears encode_scratch_bytes(nch) of it on this stream for the
    // encoder forms that use a workspace (the single-CTA forms read none of it)

    EncodeArgs a;
    memset(&a, 0, sizeof(a));
    a.x = (const uint16_t *)x;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.map.ld = ld;
    a.n_chunks = nch;
    a.chunk_base = 0;
    a.c_scale = scale_fwd(p->alpha);
    a.k = p->rice_k;
    a.k_last = k_last_of(*p);
    a.seed = p->seed;
    a.stream = d_stream;
    a.cap_words = cap_words;
    a.offsets = d_offsets;
    a.stats = d_stats;
    a.stats_add = 0;
    set_scratch(a, scratch, nch);
    a.tcols = (int)(cols / kTile);
    a.spin_limit = spin_limit();
    return launch_encode(p->lattice, p->dither, a, s) == cudaSuccess ? HQ_OK : HQ_ECUDA;
}

}  // extern "C"

static_assert(kStaticScratchBytes >= (size_t)HQ_STATIC_MAX_CHUNKS * 8 + 8 + sizeof(hq_stats),
              "scratch too small for the limit");
