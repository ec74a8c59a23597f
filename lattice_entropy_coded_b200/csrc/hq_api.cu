// hq_api.cu -- the extern "C" entry points of libhq.so (declared in hq.h):
// argument validation, workspace clearing and kernel launches.  Host code only;
// every step of the codec runs in the kernels of hq_encode.cu / hq_decode.cu.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "hq_internal.h"

using namespace hq;

namespace hq {
int g_encode_path = 0;

namespace {
constexpr int64_t kMaxCols = 65536;  // the shared sign table holds cols / 128 columns
uint32_t g_spin_limit = kSpinLimit;
bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
}  // namespace

uint32_t spin_limit() { return g_spin_limit; }

int check_params(const hq_params *p) {
    if (!p) return HQ_EINVAL;
    if (p->lattice < HQ_Z || p->lattice > HQ_E8) return HQ_EINVAL;
    if (!(p->alpha > 0.0f) || !isfinite(p->alpha)) return HQ_EINVAL;
    if (p->rice_k < 0 || p->rice_k > 15) return HQ_EINVAL;
    if (p->dither != 0 && p->dither != 1) return HQ_EINVAL;
    if (p->tile != kTile || p->chunk_tiles != kChunkTiles) return HQ_EUNSUPPORTED;
    if (p->rotation && !aligned(p->rotation, 16)) return HQ_EINVAL;
    if (p->rice_dk_last < 0 || p->rice_dk_last > 15) return HQ_EINVAL;
    return HQ_OK;
}

// Rice parameter of the last symbol of each A2 / D4 / E8 block (Z has none).
int k_last_of(const hq_params &p) {
    if (p.lattice == HQ_Z) return p.rice_k;
    return p.rice_k > p.rice_dk_last ? p.rice_k - p.rice_dk_last : 0;
}

// The weights entry points take no dense rotation (a KV-cache option).
int check_weight_params(const hq_params *p) {
    const int rc = check_params(p);
    if (rc) return rc;
    return p->rotation ? HQ_EUNSUPPORTED : HQ_OK;
}

int check_matrix(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0 || cols % kTile) return HQ_EINVAL;
    if (cols > kMaxCols) return HQ_EUNSUPPORTED;
    // at most 2^39 elements (2^27 chunks): the weights decoder's chunk arithmetic is 32-bit
    if (rows > 0 && cols > 0 && rows > (INT64_C(1) << 39) / cols) return HQ_EUNSUPPORTED;
    return HQ_OK;
}

uint64_t chunks_of(int64_t rows, int64_t cols) {
    uint64_t tiles = (uint64_t)rows * (uint64_t)(cols / kTile);
    return (tiles + kChunkTiles - 1) / kChunkTiles;
}

float scale_fwd(float alpha) { return (float)((double)alpha / sqrt(128.0)); }
float scale_inv(float alpha) { return (float)(1.0 / ((double)alpha * sqrt(128.0))); }
// With the dense rotation Q (orthonormal: no 1/sqrt(128) to fold in): u = (Q x) alpha,
// and the inverse scales by fp32(1 / alpha).
float scale_fwd_of(const hq_params &p, float alpha) { return p.rotation ? alpha : scale_fwd(alpha); }
float scale_inv_of(const hq_params &p, float alpha) {
    return p.rotation ? (float)(1.0 / (double)alpha) : scale_inv(alpha);
}

size_t ws_bytes_for(uint64_t n_chunks) {
    const size_t b = encode_scratch_bytes(n_chunks);
    return (b + 255) & ~(size_t)255;
}

// The encoder's workspace pointers (layout in hq_internal.h).
void set_scratch(EncodeArgs &a, void *ws, uint64_t nch) {
    char *b = (char *)ws;
    a.lookback = (unsigned long long *)b;
    a.ticket = (unsigned int *)(b + nch * 8);
    a.done = (unsigned int *)(b + nch * 8 + 4);
    a.acc = (hq_stats *)(b + nch * 8 + 8);
}

}  // namespace hq

namespace {

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? HQ_OK : HQ_ECUDA; }

// Per-chunk word bound for ntiles tiles with symbols <= zmax; the last symbol of each
// block (1 in n of them) takes Rice parameter kl.
uint64_t chunk_bound(int lattice, int k, int kl, uint64_t ntiles, uint64_t zmax) {
    const uint64_t n = lattice == HQ_E8 ? 8 : lattice == HQ_D4 ? 4 : lattice == HQ_A2 ? 2 : 1;
    const uint64_t nsym = ntiles * kTile, nlast = n > 1 ? nsym / n : 0;
    const uint64_t nc = (lattice == HQ_E8) ? (16 * ntiles + 31) / 32 : 0;
    const uint64_t rbits = (nsym - nlast) * (uint64_t)k + nlast * (uint64_t)kl;
    const uint64_t ubits = (nsym - nlast) * (1 + (zmax >> k)) + nlast * (1 + (zmax >> kl));
    return nc + (rbits + 31) / 32 + (ubits + 31) / 32;
}

}  // namespace

extern "C" {

int hq_stream_bound(int64_t rows, int64_t cols, const hq_params *p, uint32_t max_abs_symbol, uint64_t *max_words,
                    uint64_t *n_chunks) {
    int rc = check_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    if (!max_words || !n_chunks) return HQ_EINVAL;
    uint64_t m = max_abs_symbol ? max_abs_symbol : 255u;
    uint64_t zmax = 2 * m + 1;
    uint64_t tiles = (uint64_t)rows * (uint64_t)(cols / kTile);
    uint64_t nch = chunks_of(rows, cols);
    uint64_t full = tiles / kChunkTiles, rest = tiles % kChunkTiles;
    uint64_t words = full * chunk_bound(p->lattice, p->rice_k, k_last_of(*p), kChunkTiles, zmax);
    if (rest) words += chunk_bound(p->lattice, p->rice_k, k_last_of(*p), rest, zmax);
    *max_words = words;
    *n_chunks = nch;
    return HQ_OK;
}

int hq_workspace_bytes(uint64_t n_chunks, size_t *bytes) {
    if (!bytes) return HQ_EINVAL;
    *bytes = ws_bytes_for(n_chunks);
    return HQ_OK;
}

int hq_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, uint32_t *d_stream,
                uint64_t cap_words, uint64_t *d_offsets, hq_stats *d_stats, void *workspace, size_t ws_bytes,
                void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    const uint64_t nch = chunks_of(rows, cols);
    if (!d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (nch == 0) {
        if (d_stats && cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
        return cuda_rc(cudaMemsetAsync(d_offsets, 0, sizeof(uint64_t), s));
    }
    if (!x || !aligned(x, 16) || ld < cols || ld % 8) return HQ_EINVAL;
    if (!d_stream || !aligned(d_stream, 4)) return HQ_EINVAL;
    if (!workspace || !aligned(workspace, 8) || ws_bytes < ws_bytes_for(nch)) return HQ_EINVAL;
    // the launcher clears the workspace (look-back words, ticket, done counter, stats
    // accumulator) when the form it picks uses it; the kernel writes *d_stats

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
    set_scratch(a, workspace, nch);
    a.tcols = (int)(cols / kTile);
    a.spin_limit = g_spin_limit;
    return cuda_rc(launch_encode(p->lattice, p->dither, a, s));
}

int hq_dequantize(const uint32_t *d_stream, uint64_t stream_words, const uint64_t *d_offsets, int64_t rows,
                  int64_t cols, const hq_params *p, void *out, int out_dtype, int64_t ld, hq_stats *d_stats,
                  void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    if (out_dtype != 0 && out_dtype != 1) return HQ_EINVAL;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (d_stats && cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
    const uint64_t nch = chunks_of(rows, cols);
    if (nch == 0) return HQ_OK;
    if (!d_stream || !aligned(d_stream, 4) || !d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (!out || !aligned(out, 16) || ld < cols || ld % (out_dtype ? 4 : 8)) return HQ_EINVAL;

    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.stream = d_stream;
    a.stream_words = stream_words;
    a.offsets = d_offsets;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.n_chunks = nch;
    a.e_scale = scale_inv(p->alpha);
    a.k = p->rice_k;
    a.k_last = k_last_of(*p);
    a.seed = p->seed;
    a.out = out;
    a.out_fp32 = out_dtype;
    a.out_ld = ld;
    a.stats = d_stats;
    a.tcols = (int)(cols / kTile);
    return cuda_rc(launch_decode(p->lattice, p->dither, a, s));
}

int hq_batch_workspace_bytes(int64_t batch, uint64_t n_chunks, size_t *bytes) {
    if (!bytes || batch < 0) return HQ_EINVAL;
    if (n_chunks && (uint64_t)batch > (UINT64_C(1) << 40) / n_chunks) return HQ_EUNSUPPORTED;
    const size_t b = encode_scratch_bytes((uint64_t)batch * n_chunks, batch > 1 ? (uint64_t)batch : 1u);
    *bytes = (b + 255) & ~(size_t)255;
    return HQ_OK;
}

int hq_quantize_batch(const void *x, int64_t batch, int64_t x_stride, int64_t rows, int64_t cols, int64_t ld,
                      const hq_params *p, uint32_t *d_stream, uint64_t stream_stride, uint64_t cap_words,
                      uint64_t *d_offsets, hq_stats *d_stats, void *workspace, size_t ws_bytes, void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    if (batch < 0) return HQ_EINVAL;
    if (batch == 1)
        return hq_quantize(x, rows, cols, ld, p, d_stream, cap_words, d_offsets, d_stats, workspace, ws_bytes,
                           cuda_stream);
    const uint64_t nch = chunks_of(rows, cols);
    // chunk tickets are 32-bit counters: the whole launch stays well below 2^32 chunks
    if (batch > 0 && nch > 0 && (uint64_t)batch > (UINT64_C(1) << 31) / nch) return HQ_EUNSUPPORTED;
    if (batch == 0) return HQ_OK;
    if (!d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (nch == 0) {
        if (d_stats && cudaMemsetAsync(d_stats, 0, (size_t)batch * sizeof(hq_stats), s) != cudaSuccess)
            return HQ_ECUDA;
        // offsets[i * 1] = 0 for every item: each item's single entry
        return cuda_rc(cudaMemsetAsync(d_offsets, 0, (size_t)batch * sizeof(uint64_t), s));
    }
    if (!x || !aligned(x, 16) || ld < cols || ld % 8) return HQ_EINVAL;
    if (x_stride < 0 || x_stride % 8 || x_stride < (rows - 1) * ld + cols) return HQ_EINVAL;
    if (!d_stream || !aligned(d_stream, 4) || stream_stride < cap_words) return HQ_EINVAL;
    size_t need = 0;
    if ((rc = hq_batch_workspace_bytes(batch, nch, &need))) return rc;
    if (!workspace || !aligned(workspace, 8) || ws_bytes < need) return HQ_EINVAL;

    EncodeArgs a;
    memset(&a, 0, sizeof(a));
    a.x = (const uint16_t *)x;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.map.ld = ld;
    a.n_chunks = (uint64_t)batch * nch;
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
    set_scratch(a, workspace, a.n_chunks);
    a.tcols = (int)(cols / kTile);
    a.spin_limit = g_spin_limit;
    a.batch = (uint64_t)batch;
    a.item_chunks = nch;
    a.item_stream_stride = stream_stride;
    a.item_x_stride = x_stride;
    return cuda_rc(launch_encode(p->lattice, p->dither, a, s));
}

int hq_dequantize_batch(const uint32_t *d_stream, uint64_t stream_stride, uint64_t stream_words,
                        const uint64_t *d_offsets, int64_t batch, int64_t rows, int64_t cols, const hq_params *p,
                        void *out, int out_dtype, int64_t ld, int64_t out_stride, hq_stats *d_stats, void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    if (batch < 0) return HQ_EINVAL;
    if (batch == 1)
        return hq_dequantize(d_stream, stream_words, d_offsets, rows, cols, p, out, out_dtype, ld, d_stats,
                             cuda_stream);
    if (out_dtype != 0 && out_dtype != 1) return HQ_EINVAL;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    const uint64_t nch = chunks_of(rows, cols);
    if (batch > 0 && nch > 0 && (uint64_t)batch > (UINT64_C(1) << 27) / nch) return HQ_EUNSUPPORTED;
    if (batch == 0) return HQ_OK;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (d_stats && cudaMemsetAsync(d_stats, 0, (size_t)batch * sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
    if (nch == 0) return HQ_OK;
    if (!d_stream || !aligned(d_stream, 4) || !d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (stream_stride < stream_words) return HQ_EINVAL;
    if (!out || !aligned(out, 16) || ld < cols || ld % (out_dtype ? 4 : 8)) return HQ_EINVAL;
    if (out_stride < 0 || out_stride % (out_dtype ? 4 : 8) || out_stride < (rows - 1) * ld + cols) return HQ_EINVAL;

    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.stream = d_stream;
    a.stream_words = stream_words;
    a.offsets = d_offsets;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.n_chunks = (uint64_t)batch * nch;
    a.e_scale = scale_inv(p->alpha);
    a.k = p->rice_k;
    a.k_last = k_last_of(*p);
    a.seed = p->seed;
    a.out = out;
    a.out_fp32 = out_dtype;
    a.out_ld = ld;
    a.stats = d_stats;
    a.tcols = (int)(cols / kTile);
    a.batch = (uint64_t)batch;
    a.item_chunks = nch;
    a.item_stream_stride = stream_stride;
    a.item_out_stride = out_stride;
    return cuda_rc(launch_decode(p->lattice, p->dither, a, s));
}

int hq_gemv_workspace_bytes(int64_t rows, int64_t cols, size_t *bytes) {
    if (!bytes) return HQ_EINVAL;
    int rc = check_matrix(rows, cols);
    if (rc) return rc;
    const size_t b = (size_t)rows * (size_t)(cols / kTile) * sizeof(float);
    *bytes = (b + 255) & ~(size_t)255;
    return HQ_OK;
}

int hq_gemv(const uint32_t *d_stream, uint64_t stream_words, const uint64_t *d_offsets, int64_t rows, int64_t cols,
            const hq_params *p, const void *d_x, float *d_y, void *workspace, size_t ws_bytes, hq_stats *d_stats,
            void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if ((rc = check_matrix(rows, cols))) return rc;
    if (d_stats && !aligned(d_stats, 8)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (d_stats && cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
    if (rows == 0) return HQ_OK;
    if (!d_y || !aligned(d_y, 4)) return HQ_EINVAL;
    if (cols == 0) return cuda_rc(cudaMemsetAsync(d_y, 0, (size_t)rows * sizeof(float), s));
    if (!d_stream || !aligned(d_stream, 4) || !d_offsets || !aligned(d_offsets, 8)) return HQ_EINVAL;
    if (!d_x || !aligned(d_x, 16)) return HQ_EINVAL;
    size_t need = 0;
    hq_gemv_workspace_bytes(rows, cols, &need);
    if (!workspace || !aligned(workspace, 16) || ws_bytes < need) return HQ_EINVAL;

    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.stream = d_stream;
    a.stream_words = stream_words;
    a.offsets = d_offsets;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.n_chunks = chunks_of(rows, cols);
    a.e_scale = scale_inv(p->alpha);
    a.k = p->rice_k;
    a.k_last = k_last_of(*p);
    a.seed = p->seed;
    a.out = nullptr;
    a.stats = d_stats;
    a.tcols = (int)(cols / kTile);
    a.vec = (const uint16_t *)d_x;
    a.res = (float *)workspace;
    return cuda_rc(launch_gemv(p->lattice, p->dither, a, d_y, s));
}

int hq_kv_init(hq_kv_cache *cache, int32_t heads, int32_t head_dim, const hq_params *p, uint32_t *d_words,
               uint64_t cap_words, uint64_t *d_offsets, uint64_t offsets_cap, hq_kv_append_row *d_table,
               uint64_t table_cap, uint64_t *d_tail, hq_stats *d_stats, void *cuda_stream) {
    if (!cache || !p) return HQ_EINVAL;
    if (p->lattice < HQ_Z || p->lattice > HQ_E8 || p->rice_k < 0 || p->rice_k > 15) return HQ_EINVAL;
    if (p->dither != 0 && p->dither != 1) return HQ_EINVAL;
    if (p->tile != kTile || p->chunk_tiles != kChunkTiles) return HQ_EUNSUPPORTED;
    if (p->rotation && !aligned(p->rotation, 16)) return HQ_EINVAL;
    if (p->rice_dk_last < 0 || p->rice_dk_last > 15) return HQ_EINVAL;
    if (head_dim != kTile) return HQ_EUNSUPPORTED;
    if (heads <= 0) return HQ_EINVAL;
    if (!d_words || !aligned(d_words, 4) || !d_offsets || !aligned(d_offsets, 8) || offsets_cap < 1) return HQ_EINVAL;
    if (!d_table || !aligned(d_table, 8) || table_cap < 1 || !d_tail || !aligned(d_tail, 8)) return HQ_EINVAL;
    if (!d_stats || !aligned(d_stats, 8)) return HQ_EINVAL;
    memset(cache, 0, sizeof(*cache));
    cache->d_words = d_words;
    cache->cap_words = cap_words;
    cache->d_offsets = d_offsets;
    cache->offsets_cap = offsets_cap;
    cache->d_table = d_table;
    cache->table_cap = table_cap;
    cache->d_tail = d_tail;
    cache->d_stats = d_stats;
    cache->heads = heads;
    cache->head_dim = head_dim;
    cache->params = *p;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    if (cudaMemsetAsync(d_tail, 0, 2 * sizeof(uint64_t), s) != cudaSuccess) return HQ_ECUDA;
    if (cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
    if (cudaMemsetAsync(d_offsets, 0, sizeof(uint64_t), s) != cudaSuccess) return HQ_ECUDA;
    return HQ_OK;
}

int hq_kv_append(hq_kv_cache *cache, const void *kv, int64_t T, int64_t ld_token, int64_t ld_head, float alpha,
                 void *workspace, size_t ws_bytes, void *cuda_stream) {
    if (!cache || !cache->d_words) return HQ_EINVAL;
    hq_params p = cache->params;
    p.alpha = alpha;
    int rc = check_params(&p);
    if (rc) return rc;
    if (T < 0) return HQ_EINVAL;
    if (T == 0) return HQ_OK;
    if (!kv || !aligned(kv, 16) || ld_token < kTile || ld_token % 8 || ld_head % 8 || ld_head < 0) return HQ_EINVAL;
    const uint64_t H = (uint64_t)cache->heads;
    const uint64_t nch = H * (uint64_t)((T + 31) / 32);
    if (cache->chunks + nch + 1 > cache->offsets_cap || cache->appends + 1 > cache->table_cap) return HQ_EINVAL;
    if (!workspace || !aligned(workspace, 8) || ws_bytes < ws_bytes_for(nch)) return HQ_EINVAL;
    cudaStream_t s = (cudaStream_t)cuda_stream;
    EncodeArgs a;
    memset(&a, 0, sizeof(a));
    a.x = (const uint16_t *)kv;
    a.map.kv = 1;
    a.map.heads = (int64_t)H;
    a.map.tokens = T;
    a.map.ld_tok = ld_token;
    a.map.ld_head = ld_head;
    a.map.tok0 = cache->tokens;
    a.n_chunks = nch;
    a.chunk_base = cache->chunks;
    a.c_scale = scale_fwd_of(p, alpha);
    a.k = p.rice_k;
    a.k_last = k_last_of(p);
    a.seed = p.seed;
    a.rot = p.rotation;
    a.stream = cache->d_words;
    a.cap_words = cache->cap_words;
    a.offsets = cache->d_offsets;
    a.base_ptr = cache->d_tail + (cache->appends & 1);
    a.tail_out = cache->d_tail + ((cache->appends + 1) & 1);
    a.row = cache->d_table + cache->appends;
    a.row_val.first_chunk = cache->chunks;
    a.row_val.token0 = cache->tokens;
    a.row_val.tokens = (int32_t)T;
    a.row_val.alpha = alpha;
    a.row_val.scale_fwd = a.c_scale;
    a.row_val.scale_inv = scale_inv_of(p, alpha);
    a.stats = cache->d_stats;
    a.stats_add = 1;
    set_scratch(a, workspace, nch);
    a.tcols = 1;
    a.spin_limit = g_spin_limit;
    rc = cuda_rc(launch_encode(p.lattice, p.dither, a, s));
    if (rc) return rc;
    cache->tokens += T;
    cache->chunks += nch;
    cache->appends += 1;
    return HQ_OK;
}

int hq_kv_read(const hq_kv_cache *cache, void *out, int out_dtype, int64_t len, int64_t out_ld_token,
               int64_t out_ld_head, void *cuda_stream) {
    if (!cache || !cache->d_words) return HQ_EINVAL;
    if (out_dtype != 0 && out_dtype != 1) return HQ_EINVAL;
    if (len < 0 || len > cache->tokens) return HQ_EINVAL;
    if (len == 0 || cache->chunks == 0) return HQ_OK;
    const int m = out_dtype ? 4 : 8;
    if (!out || !aligned(out, 16) || out_ld_token < kTile || out_ld_token % m || out_ld_head % m || out_ld_head < 0)
        return HQ_EINVAL;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.stream = cache->d_words;
    a.stream_words = cache->cap_words;
    a.offsets = cache->d_offsets;
    a.map.kv = 1;
    a.map.heads = cache->heads;
    a.n_chunks = cache->chunks;
    a.k = cache->params.rice_k;
    a.k_last = k_last_of(cache->params);
    a.seed = cache->params.seed;
    a.out = out;
    a.out_fp32 = out_dtype;
    a.out_ld = out_ld_token;
    a.out_ld_head = out_ld_head;
    a.len = len;
    a.table = cache->d_table;
    a.n_appends = cache->appends;
    a.stats = cache->d_stats;
    a.tcols = 1;
    a.rot = cache->params.rotation;
    return cuda_rc(launch_decode(cache->params.lattice, cache->params.dither, a, (cudaStream_t)cuda_stream));
}

// ------------------------------------------------------------------ rate and calibration
}  // extern "C"

namespace {

// Rate-only launch over the tile map in `a` (weights or KV), stats zeroed first.
int rate_launch(const hq_params *p, EncodeArgs &a, hq_stats *d_stats, cudaStream_t s) {
    if (cudaMemsetAsync(d_stats, 0, sizeof(hq_stats), s) != cudaSuccess) return HQ_ECUDA;
    if (a.n_chunks == 0) return HQ_OK;
    a.c_scale = scale_fwd_of(*p, p->alpha);
    a.k = p->rice_k;
    a.k_last = k_last_of(*p);
    a.seed = p->seed;
    a.rot = p->rotation;
    a.stats = d_stats;
    return cuda_rc(launch_rate(p->lattice, p->dither, a, s));
}

int weights_rate_args(const void *x, int64_t rows, int64_t cols, int64_t ld, EncodeArgs &a) {
    int rc = check_matrix(rows, cols);
    if (rc) return rc;
    memset(&a, 0, sizeof(a));
    a.n_chunks = chunks_of(rows, cols);
    if (a.n_chunks && (!x || !aligned(x, 16) || ld < cols || ld % 8)) return HQ_EINVAL;
    a.x = (const uint16_t *)x;
    a.map.kv = 0;
    a.map.rows = rows;
    a.map.cols = cols;
    a.map.ld = ld;
    a.tcols = (int)(cols / kTile);
    return HQ_OK;
}

int kv_rate_args(const void *kv, int32_t heads, int64_t T, int64_t ld_token, int64_t ld_head, int64_t tok0,
                 EncodeArgs &a) {
    if (heads <= 0 || T < 0 || tok0 < 0) return HQ_EINVAL;
    memset(&a, 0, sizeof(a));
    a.n_chunks = (uint64_t)heads * (uint64_t)((T + 31) / 32);
    if (a.n_chunks && (!kv || !aligned(kv, 16) || ld_token < kTile || ld_token % 8 || ld_head % 8 || ld_head < 0))
        return HQ_EINVAL;
    a.x = (const uint16_t *)kv;
    a.map.kv = 1;
    a.map.heads = heads;
    a.map.tokens = T;
    a.map.ld_tok = ld_token;
    a.map.ld_head = ld_head;
    a.map.tok0 = tok0;
    a.tcols = 1;
    return HQ_OK;
}

int check_spec(const hq_calib_spec *sp) {
    if (!sp) return HQ_EINVAL;
    if (!(sp->target_bps > 0.0) || !(sp->tol >= 0.0) || !(sp->alpha_lo > 0.0) || !(sp->alpha_hi > sp->alpha_lo) ||
        !isfinite(sp->alpha_hi) || !isfinite(sp->target_bps))
        return HQ_EINVAL;
    if (sp->k_lo < 0 || sp->k_hi > 15 || sp->k_lo > sp->k_hi || sp->max_iter < 0 || sp->max_iter > 200)
        return HQ_EINVAL;
    return HQ_OK;
}

// Payload bits per scalar at (alpha, k): one rate launch, copied back and waited for.
// A launch that flags HQ_ST_RANGE counts as +infinity (the rate only grows with alpha).
int rate_at(const hq_params &base, float alpha, int k, EncodeArgs a, double n, hq_stats *d_stats, cudaStream_t s,
            double &bps, uint32_t &seen) {
    hq_params p = base;
    p.alpha = alpha;
    p.rice_k = k;
    int rc = rate_launch(&p, a, d_stats, s);
    if (rc) return rc;
    hq_stats h;
    if (cudaMemcpyAsync(&h, d_stats, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return HQ_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HQ_ECUDA;
    seen |= h.status;
    bps = (h.status & HQ_ST_RANGE) ? INFINITY : (double)h.payload_bits / n;
    return HQ_OK;
}

// For each k in [k_lo, k_hi]: if rate(lo) <= target <= rate(hi), bisect alpha at the
// geometric mid point until |rate - target| <= tol (at most max_iter steps; then the
// mid point of the last bracket).  The k with the largest alpha wins (the first on ties).
int calibrate(const hq_params *p, const hq_calib_spec *sp, const EncodeArgs &a, double n, hq_stats *d_stats,
              cudaStream_t s, hq_calib_result *out) {
    int rc = check_params(p);
    if (rc) return rc;
    if ((rc = check_spec(sp))) return rc;
    if (!out || !d_stats || !aligned(d_stats, 8)) return HQ_EINVAL;
    memset(out, 0, sizeof(*out));
    out->k = -1;
    if (a.n_chunks == 0) return HQ_EINVAL;
    bool found = false;
    double best = 0.0;
    for (int k = sp->k_lo; k <= sp->k_hi; k++) {
        double lo = sp->alpha_lo, hi = sp->alpha_hi, rlo, rhi, r, mid;
        if ((rc = rate_at(*p, (float)lo, k, a, n, d_stats, s, rlo, out->status))) return rc;
        if ((rc = rate_at(*p, (float)hi, k, a, n, d_stats, s, rhi, out->status))) return rc;
        out->evaluations += 2;
        if (!(rlo <= sp->target_bps && sp->target_bps <= rhi)) continue;
        bool done = false;
        for (int it = 0; it < sp->max_iter && !done; it++) {
            mid = sqrt(lo * hi);
            if ((rc = rate_at(*p, (float)mid, k, a, n, d_stats, s, r, out->status))) return rc;
            out->evaluations++;
            if (fabs(r - sp->target_bps) <= sp->tol) done = true;
            else if (r < sp->target_bps) lo = mid;
            else hi = mid;
        }
        if (!done) {
            mid = sqrt(lo * hi);
            if ((rc = rate_at(*p, (float)mid, k, a, n, d_stats, s, r, out->status))) return rc;
            out->evaluations++;
        }
        if (!found || mid > best) {
            found = true;
            best = mid;
            out->alpha = (float)mid;
            out->k = k;
            out->bps = r;
        }
    }
    return found ? HQ_OK : HQ_EUNSUPPORTED;
}

}  // namespace

extern "C" {

int hq_rate(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, hq_stats *d_stats,
            void *cuda_stream) {
    int rc = check_weight_params(p);
    if (rc) return rc;
    if (!d_stats || !aligned(d_stats, 8)) return HQ_EINVAL;
    EncodeArgs a;
    if ((rc = weights_rate_args(x, rows, cols, ld, a))) return rc;
    return rate_launch(p, a, d_stats, (cudaStream_t)cuda_stream);
}

int hq_rate_kv(const void *kv, int32_t heads, int64_t T, int64_t ld_token, int64_t ld_head, int64_t tok0,
               const hq_params *p, hq_stats *d_stats, void *cuda_stream) {
    int rc = check_params(p);
    if (rc) return rc;
    if (!d_stats || !aligned(d_stats, 8)) return HQ_EINVAL;
    EncodeArgs a;
    if ((rc = kv_rate_args(kv, heads, T, ld_token, ld_head, tok0, a))) return rc;
    return rate_launch(p, a, d_stats, (cudaStream_t)cuda_stream);
}

int hq_calibrate(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, const hq_calib_spec *spec,
                 hq_stats *d_stats, void *cuda_stream, hq_calib_result *out) {
    EncodeArgs a;
    int rc = weights_rate_args(x, rows, cols, ld, a);
    if (rc) return rc;
    if (p && p->rotation) return HQ_EUNSUPPORTED;
    return calibrate(p, spec, a, (double)rows * (double)cols, d_stats, (cudaStream_t)cuda_stream, out);
}

int hq_calibrate_kv(const void *kv, int32_t heads, int64_t T, int64_t ld_token, int64_t ld_head, int64_t tok0,
                    const hq_params *p, const hq_calib_spec *spec, hq_stats *d_stats, void *cuda_stream,
                    hq_calib_result *out) {
    EncodeArgs a;
    int rc = kv_rate_args(kv, heads, T, ld_token, ld_head, tok0, a);
    if (rc) return rc;
    return calibrate(p, spec, a, (double)heads * (double)T * kTile, d_stats, (cudaStream_t)cuda_stream, out);
}

int hq_kv_scores(const hq_kv_cache *cache, const void *d_q, int32_t group, float *d_scores, int64_t len,
                 int64_t scores_ld, void *cuda_stream) {
    if (!cache || !cache->d_words) return HQ_EINVAL;
    if (group < 1 || len < 0 || len > cache->tokens) return HQ_EINVAL;
    if (len == 0 || cache->chunks == 0) return HQ_OK;
    if (!d_q || !aligned(d_q, 16) || !d_scores || !aligned(d_scores, 4) || scores_ld < len) return HQ_EINVAL;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.stream = cache->d_words;
    a.stream_words = cache->cap_words;
    a.offsets = cache->d_offsets;
    a.map.kv = 1;
    a.map.heads = cache->heads;
    a.n_chunks = cache->chunks;
    a.k = cache->params.rice_k;
    a.k_last = k_last_of(cache->params);
    a.seed = cache->params.seed;
    a.out = nullptr;
    a.out_ld = scores_ld;
    a.len = len;
    a.table = cache->d_table;
    a.n_appends = cache->appends;
    a.stats = cache->d_stats;
    a.tcols = 1;
    a.vec = (const uint16_t *)d_q;
    a.res = d_scores;
    a.group = group;
    a.rot = cache->params.rotation;
    return cuda_rc(launch_kv_scores(cache->params.lattice, cache->params.dither, a, (cudaStream_t)cuda_stream));
}

const char *hq_status_string(int code) {
    switch (code) {
    case HQ_OK: return "ok";
    case HQ_EINVAL: return "invalid argument";
    case HQ_EUNSUPPORTED: return "unsupported by this library";
    case HQ_ECUDA: return "CUDA error";
    }
    if (code > 0) {
        if (code & HQ_ST_TIMEOUT) return "look-back timed out";
        if (code & HQ_ST_CORRUPT) return "corrupt stream";
        if (code & HQ_ST_CAPACITY) return "stream capacity exceeded";
        if (code & HQ_ST_RANGE) return "value outside the supported range";
    }
    return "unknown";
}

int hq_device_check(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ECUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return HQ_ECUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return HQ_ECUDA;
    return (major == 10 && minor == 0) ? HQ_OK : HQ_EUNSUPPORTED;
}

int hq_haar_rotation(uint64_t seed, float *d_q, void *cuda_stream) {
    if (!d_q || !aligned(d_q, 16)) return HQ_EINVAL;
    return cuda_rc(launch_haar(seed, d_q, (cudaStream_t)cuda_stream));
}

void hq_debug_set_spin_limit(uint32_t polls) { g_spin_limit = polls ? polls : kSpinLimit; }

int hq_debug_set_encode_path(int path) {
    if (path < 0 || path > 4) return HQ_EINVAL;
    hq::g_encode_path = path;
    return HQ_OK;
}

}  // extern "C"
