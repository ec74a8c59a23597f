// hq_internal.h -- launch arguments shared by the host entry points (hq_api.cu)
// and the kernels (hq_encode.cu, hq_decode.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "hq.h"

namespace hq {

constexpr int kTile = 128;          // elements per RHT tile
constexpr int kChunkTiles = 32;     // tiles per chunk (the stream's unit: one offset per chunk)
constexpr int kSignWords = 4;       // shared sign-table words per tile column (one per 32-column quarter)
constexpr int kWarpsPerCta = 8;     // warps per CTA of the per-warp and grouped encoders and the decoder
constexpr int kStageWords = 1024;   // shared staging for one chunk's words (encode and decode);
                                    // larger chunks are written or read in place in global memory
constexpr int kLanesPerTile = 4;    // lanes sharing one tile (32 elements each), except the wide encoder
constexpr int kTilesPerRound = 32 / kLanesPerTile;  // tiles a warp transforms at once; 4 rounds per chunk
constexpr uint32_t kSpinLimit = 1u << 22;   // look-back polls before giving up (HQ_ST_TIMEOUT)
constexpr uint32_t kMaxUnaryBits = 1u << 31; // chunks with more unary bits are outside the supported range

// Encoder workspace of n chunks: look-back words [0, 8n), ticket at 8n, done counter at
// 8n + 4, stats accumulator at 8n + 8 (one per item of a batch); all cleared by one memset
// of encode_scratch_bytes(n, items).
inline size_t encode_scratch_bytes(uint64_t n_chunks, uint64_t items = 1) {
    return (size_t)n_chunks * 8 + 8 + (size_t)items * sizeof(hq_stats);
}

// Salts xor-ed into the seed: "SIGN" for the sign diagonal, "DITH" for the dither.
constexpr uint64_t kSignSalt = 0x5349474Eull;
constexpr uint64_t kDitherSalt = 0x44495448ull;

// How a chunk index maps to tiles.
//  weights: chunk c = tiles [32c, 32c+32) of the row-major tile order of an R x C matrix.
//  kv     : chunk c of an append = head c / cph, tokens [32 (c % cph), ...), cph = ceil(T/32).
struct TileMap {
    int kv;
    int64_t rows, cols, ld;           // weights
    int64_t heads, tokens, ld_tok, ld_head, tok0;  // kv
};

struct EncodeArgs {
    const uint16_t *x;
    TileMap map;
    uint64_t n_chunks;        // chunks of this call
    uint64_t chunk_base;      // global index of this call's first chunk (offset array position)
    float c_scale;            // alpha / sqrt(128), rounded to fp32 on the host
    int k;                    // Rice parameter
    int k_last;               // Rice parameter of the last symbol of each A2 / D4 / E8 block (k: single code)
    uint64_t seed;
    uint32_t *stream;
    uint64_t cap_words;
    uint64_t *offsets;        // offsets[chunk_base + c] written for c in [0, n_chunks]
    const uint64_t *base_ptr; // device word index where this call's stream starts (KV tail) or null (0)
    uint64_t *tail_out;       // device word updated with the end of this call's stream, or null
    hq_kv_append_row *row;    // KV: table row written by the warp of chunk 0, or null
    hq_kv_append_row row_val;
    hq_stats *stats;          // the caller's stats, or null
    int stats_add;            // 1: add this call's stats to *stats (a KV cache's running stats); 0: replace
    unsigned long long *lookback;  // n_chunks words, zeroed
    unsigned int *ticket;          // one word, zeroed
    unsigned int *done;            // one word, zeroed: CTAs finished
    hq_stats *acc;                 // zeroed: this call's stats, moved to *stats by the last CTA
    int tcols;                // tile columns in the sign table (cols / 128, or 1 for KV)
    uint32_t spin_limit;
    const float *rot;         // KV: the dense rotation Q (128 x 128 fp32, row-major) or null (sign diagonal, H_128)
    // A strided batch (hq_quantize_batch; 0 or 1: one matrix): item i of `batch` equally
    // shaped matrices is chunks [i item_chunks, (i + 1) item_chunks) of the launch; its input
    // starts i item_x_stride elements after x, its stream i item_stream_stride words after
    // stream (cap_words each), its offsets i (item_chunks + 1) entries after offsets, its
    // stats and workspace accumulator i entries after stats and acc.  The per-warp form only.
    uint64_t batch, item_chunks, item_stream_stride;
    int64_t item_x_stride;
};

struct DecodeArgs {
    const uint32_t *stream;
    uint64_t stream_words;
    const uint64_t *offsets;
    TileMap map;              // for KV the per-append fields come from the table
    uint64_t n_chunks;
    float e_scale;            // 1 / (alpha sqrt(128)), weights path
    int k;
    int k_last;               // as EncodeArgs::k_last
    uint64_t seed;
    void *out;
    int out_fp32;
    int64_t out_ld;           // weights: row stride; kv: token stride
    int64_t out_ld_head;      // kv: head stride
    int64_t len;              // kv: tokens to write
    const hq_kv_append_row *table;  // kv: append table
    uint64_t n_appends;
    hq_stats *stats;
    int tcols;
    // dot-product outputs (hq_gemv, hq_kv_scores) instead of stored tiles
    const uint16_t *vec;      // bf16 x [cols] (gemv) or queries [heads * group, 128] (scores)
    float *res;               // gemv: one partial per tile [rows * tcols]; scores: [heads * group, out_ld]
    int group;                // scores: query heads per KV head
    const float *rot;         // KV: the dense rotation Q, or null
    // A strided batch (hq_dequantize_batch; 0 or 1: one matrix): chunk c of the launch is
    // chunk c mod item_chunks of item c / item_chunks, whose stream starts i item_stream_stride
    // words after stream (stream_words each), offsets i (item_chunks + 1) entries after
    // offsets, output i item_out_stride elements after out, stats i entries after stats.
    // Stored tiles only.
    uint64_t batch, item_chunks, item_stream_stride;
    int64_t item_out_stride;
};

// Decoder outputs: the tile itself, its dot product with x, or its dot products with queries.
// kStoreTiles stores bf16 or fp32 (DecodeArgs::out_fp32); kStoreBf16 stores bf16 only
// (the fp32 store compiled out).
enum DecodeMode { kStoreTiles = 0, kGemvPartials = 1, kKvScores = 2, kStoreBf16 = 3 };

// Persistent-grid size of one kernel on the current device: SM count x resident CTAs per SM at
// `smem` dynamic shared bytes, capped at `want` CTAs.  The shared-memory attribute and the
// occupancy query run once per device and shared-memory size; later calls of the same kernel
// (every KV append, every small matrix) reuse the cached answer.
struct LaunchPlan {
    static constexpr int kMaxDevices = 64;
    std::mutex mu;
    int sms[kMaxDevices] = {};
    size_t configured[kMaxDevices] = {};   // dynamic shared bytes the attribute allows
    size_t smem_key[kMaxDevices] = {};
    int per_sm[kMaxDevices] = {};

    template <typename K>
    cudaError_t grid(K kern, int threads, size_t smem, unsigned long long want, unsigned &out) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lk(mu);
        if (!sms[dev] && (e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if (smem > configured[dev]) {
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return e;
            configured[dev] = smem;
        }
        if (smem_key[dev] != smem || per_sm[dev] == 0) {
            int n = 0;
            if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem)) != cudaSuccess) return e;
            if (n < 1) return cudaErrorInvalidConfiguration;
            smem_key[dev] = smem;
            per_sm[dev] = n;
        }
        unsigned long long g = (unsigned long long)sms[dev] * (unsigned long long)per_sm[dev];
        if (want < g) g = want;
        out = (unsigned)(g < 1 ? 1 : g);
        return cudaSuccess;
    }
};

// Host-side argument checks and launch values shared by the entry points (hq_api.cu,
// hq_static.cu), so that every entry point applies the same rules.
int check_params(const hq_params *p);          // HQ_OK, HQ_EINVAL or HQ_EUNSUPPORTED
int check_weight_params(const hq_params *p);   // check_params, and no dense rotation
int check_matrix(int64_t rows, int64_t cols);  // cols % 128, cols <= 65536, rows * cols <= 2^40
uint64_t chunks_of(int64_t rows, int64_t cols);
int k_last_of(const hq_params &p);             // Rice parameter of the last symbol of a block
float scale_fwd(float alpha);                  // fp32(alpha / sqrt(128))
void set_scratch(EncodeArgs &a, void *ws, uint64_t nch);   // look-back, ticket, done, stats pointers
uint32_t spin_limit();                         // look-back polls (hq_debug_set_spin_limit)

// Encoder form: 0 = by size (one CTA for a few chunks, then wide, then grouped, for
// launches of fewer chunks than the per-warp form has resident warps, per-warp otherwise), 1 =
// per-warp, 2 = grouped (4 warps per chunk), 3 = wide (16 warps per chunk, 16 lanes
// per tile), 4 = one CTA.  Set by hq_debug_set_encode_path (hq_api.cu); all forms
// give identical streams.
extern int g_encode_path;

// Launchers (defined in hq_encode.cu / hq_decode.cu).  Return cudaSuccess or the launch error.
cudaError_t launch_encode(int lattice, int dither, const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_decode(int lattice, int dither, const DecodeArgs &a, cudaStream_t s);
// hq_gemv: per-tile partials into a.res, then y[r] = sum of row r's partials in column order.
cudaError_t launch_gemv(int lattice, int dither, const DecodeArgs &a, float *y, cudaStream_t s);
// hq_kv_scores: a.res[(h * group + g) * out_ld + t] for every cached token t < len.
cudaError_t launch_kv_scores(int lattice, int dither, const DecodeArgs &a, cudaStream_t s);
// Rate only: adds payload_bits, stream_words, max_symbol and HQ_ST_RANGE of the call into a.stats
// (zeroed by the caller); reads a.x, a.map, a.n_chunks, a.c_scale, a.k, a.seed, a.tcols.
cudaError_t launch_rate(int lattice, int dither, const EncodeArgs &a, cudaStream_t s);
// The same with the dense KV rotation a.rot (hq_rot_encode.cu, hq_rot_decode.cu); the launchers
// above forward to these when a.rot is set.
cudaError_t launch_encode_rot(int lattice, int dither, const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_rate_rot(int lattice, int dither, const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_decode_rot(int lattice, int dither, const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_kv_scores_rot(int lattice, int dither, const DecodeArgs &a, cudaStream_t s);
// Haar-uniform rotation for the seed (hq_haar.cu): one CTA, q = 128 x 128 fp32 row-major.
cudaError_t launch_haar(uint64_t seed, float *q, cudaStream_t s);

}  // namespace hq
