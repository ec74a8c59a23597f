// hq_static.cu -- hq_quantize_static: the weights-path quantize + encode for
// callers that cannot allocate device memory.  The encoder's scratch (the
// chunk look-back words and the chunk ticket) lives in a fixed array that is
// part of this library's device image instead of in a caller workspace.
//
// The array is a host-side stand-in in host code: its address on a device is
// obtained once per device with cudaGetSymbolAddress (with that device
// current) and cached; kernels receive that device address.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "hq_internal.h"

using namespace hq;

namespace {

constexpr size_t kStaticScratchBytes = HQ_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Look-back words (8 bytes per chunk), the ticket and done words, the stats accumulator.
static __device__ __align__(256) unsigned char g_hq_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_addr[kMaxDevices];   // device address of g_hq_scratch per device, null until set up

// Device address of the scratch on the current device (set up on first use).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return HQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_hq_scratch) != cudaSuccess || !p) return HQ_ECUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return HQ_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" {

int hq_quantize_static(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, uint32_t *d_stream,
                       uint64_t cap_words, uint64_t *d_offsets, hq_stats *d_stats, void *cuda_stream) {
    if (!p) return HQ_EINVAL;
    if (p->lattice < HQ_Z || p->lattice > HQ_E8) return HQ_EINVAL;
    if (!(p->alpha > 0.0f) || !(p->alpha < __builtin_inff())) return HQ_EINVAL;
    if (p->rice_k < 0 || p->rice_k > 15 || (p->dither != 0 && p->dither != 1)) return HQ_EINVAL;
    if (p->tile != kTile || p->chunk_tiles != kChunkTiles) return HQ_EUNSUPPORTED;
    if (p->rotation) return HQ_EUNSUPPORTED;   // the dense rotation is a KV-cache option
    if (p->rice_dk_last < 0 || p->rice_dk_last > 15) return HQ_EINVAL;
    if (rows < 0 || cols < 0 || cols % kTile) return HQ_EINVAL;
    if (cols > 65536) return HQ_EUNSUPPORTED;
    const uint64_t tiles = (uint64_t)rows * (uint64_t)(cols / kTile);
    const uint64_t nch = (tiles + kChunkTiles - 1) / kChunkTiles;
    if (nch > HQ_STATIC_MAX_CHUNKS) return HQ_EUNSUPPORTED;   // beyond the fixed scratch
    if (!d_offsets || !aligned(d_offsets, 8) || (d_stats && !aligned(d_stats, 8))) return HQ_EINVAL;
    void *scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc) return rc;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (nch == 0) {
        if (d_stats && cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
        return cudaMemsetAsync(d_offsets, 0, sizeof(uint64_t), s) == cudaSuccess ? HQ_OK : HQ_ECUDA;
    }
    if (!x || !aligned(x, 16) || ld < cols || ld % 8) return HQ_EINVAL;
    if (!d_stream || !aligned(d_stream, 4)) return HQ_EINVAL;
    // the previous call's look-back words, ticket, counter and stats are still there:
    // clear what this call uses

    EncodeArgs a;
    memset(&a, 0, sizeof(a));
    a.x = (const uint16_t *)x;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.map.ld = ld;
    a.n_chunks = nch;
    a.chunk_base = 0;
    a.c_scale = (float)((double)p->alpha / __builtin_sqrt(128.0));
    a.k = p->rice_k;
    a.k_last = (p->lattice == HQ_Z) ? p->rice_k : (p->rice_k > p->rice_dk_last ? p->rice_k - p->rice_dk_last : 0);
    a.seed = p->seed;
    a.stream = d_stream;
    a.cap_words = cap_words;
    a.offsets = d_offsets;
    a.stats = d_stats;
    a.stats_add = 0;
    a.lookback = (unsigned long long *)scratch;
    a.ticket = (unsigned int *)((char *)scratch + nch * 8);
    a.done = (unsigned int *)((char *)scratch + nch * 8 + 4);
    a.acc = (hq_stats *)((char *)scratch + nch * 8 + 8);
    a.tcols = (int)(cols / kTile);
    a.spin_limit = kSpinLimit;
    return launch_encode(p->lattice, p->dither, a, s) == cudaSuccess ? HQ_OK : HQ_ECUDA;
}

}  // extern "C"

static_assert(kStaticScratchBytes >= (size_t)HQ_STATIC_MAX_CHUNKS * 8 + 8 + sizeof(hq_stats),
              "scratch too small for the limit");
