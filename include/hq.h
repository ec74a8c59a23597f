/*
 * hq.h -- C ABI of the B200 (sm_100a) HyperQuant codec library, libhq.so.
 *
 * The method: HyperQuant ("Hadamard, optimallY Packing, Entropy Rice-coding"),
 * as summarised on the gist.science explainer pages of paper 2606.23406
 * ("Methodology": 1 per-tile RHT, 2 lattice quantization, 3 bit-stripping and
 * Rice coding, 4 KV-cache bias correction) and its arXiv abstract (steps
 * (i)-(iv)).  Per 128-element tile: x -> D x (seeded random signs) -> H_128
 * (Walsh-Hadamard) -> scale by alpha / sqrt(128) -> [+ dither d] -> nearest
 * point of the lattice (Z, A2, D4 or E8 in an integer embedding) -> strip the
 * membership-implied bits -> zigzag -> Rice code with parameter k into a
 * chunked bitstream.  The inverse undoes every step.  A KV cache may instead
 * rotate each token's head vector by a full Haar-uniform 128 x 128 orthogonal
 * matrix ("Methodology" 4: a per-layer rotation, full Haar-uniform or the cheap
 * sign diagonal); see hq_params.rotation and hq_haar_rotation.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer named d_* or documented as "device" is device memory of the
 *    current CUDA device; host pointers are named h_* or documented as host.
 *  - The caller owns all memory.  The library allocates nothing, and every call
 *    is asynchronous on the CUDA stream it is given (a cudaStream_t passed as
 *    void*; NULL = legacy default stream), except hq_calibrate and
 *    hq_calibrate_kv, which wait for each of their rate passes.
 *  - A negative return value is a synchronous argument or launch error
 *    (HQ_EINVAL, HQ_EUNSUPPORTED, HQ_ECUDA); nothing was enqueued.  Errors that
 *    depend on the data are reported on the device in hq_stats.status, which
 *    the caller reads after its own synchronisation.
 *  - bf16 tensors are little-endian IEEE bfloat16, 16-byte aligned, with
 *    element strides that are multiples of 8 elements (16 bytes).
 *  - A tile is 128 consecutive elements of a row; a chunk is 32 consecutive
 *    tiles (4096 elements).  A weights matrix (or a strided batch of them, per
 *    launch) has at most 2^27 chunks (2^39 elements, more than device memory
 *    holds); larger requests return HQ_EUNSUPPORTED.  Weights: tiles in row-major order of an R x C
 *    matrix (C % 128 == 0), chunk c = tiles [32c, 32c+32).  KV cache: per
 *    append of T tokens and H heads, ceil(T/32) chunks per head, head-major;
 *    one tile = one token's 128-dim head vector.
 *
 * Bitstream (all planes LSB-first in little-endian uint32 words, each plane
 * starting on a word boundary), per chunk of n tiles (N = 128 n symbols):
 *   [coset plane, E8 only: one bit per 8-element block, ceil(16 n / 32) words]
 *   [remainder plane: k bits per symbol at bit i*k, 4 k n words; with
 *    rice_dk_last > 0, symbol i's k_i bits at the running sum of the k_i]
 *   [unary plane: per symbol floor(z / 2^k_i) zeros then a one, zero padded]
 * offsets[c] is the index of chunk c's first word; offsets[n_chunks] is the
 * total.  The codewords are exactly the concatenated Rice codewords of the
 * symbols; the plane split lets a decoder work on all tiles of a chunk at once.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points keep default visibility (the library is built with
 * hidden visibility for everything else). */
#if defined(__GNUC__)
#define HQ_API __attribute__((visibility("default")))
#else
#define HQ_API
#endif

/* Lattices (page section "lattice quantization": E8, D4, A2 or scalar Z) in
 * their integer embeddings:
 *   HQ_Z  : Z, code q stands for q.
 *   HQ_A2 : code (a, b), a = b (mod 2), stands for (a/2, b*sqrt(3)/2)
 *           (A2 at unit minimum distance).
 *   HQ_D4 : {q in Z^4 : sum q even}.
 *   HQ_E8 : 2E8 = 2D8 u (2D8 + 1) in Z^8 (all coordinates of one parity, and
 *           (q - parity)/2 has an even sum). */
enum hq_lattice { HQ_Z = 0, HQ_A2 = 1, HQ_D4 = 2, HQ_E8 = 3 };

/* Synchronous return codes. */
#define HQ_OK 0
#define HQ_EINVAL (-1)       /* bad argument: null pointer, size, stride, alignment, parameter */
#define HQ_EUNSUPPORTED (-2) /* valid request outside what this library supports (tile != 128, ...) */
#define HQ_ECUDA (-3)        /* a CUDA launch or runtime call failed */

/* Device-side status bits (hq_stats.status). */
#define HQ_ST_CAPACITY 0x1u /* the stream needs more than cap_words words: words at or past the cap
                               were not written; stats.stream_words holds the size needed */
#define HQ_ST_CORRUPT 0x2u  /* a chunk failed a consistency check while decoding (offsets out of range
                               or not monotone, wrong number of unary terminators); its tiles are zero */
#define HQ_ST_TIMEOUT 0x4u  /* the chunk-offset look-back gave up after its spin limit */
#define HQ_ST_RANGE 0x8u    /* a scaled coordinate was at or beyond 2^21 in magnitude (or not finite):
                               codes of that call are outside the supported range and unspecified */

/* Parameters of one call (page sections 1-4).  tile and chunk_tiles are
 * fixed in this library; the others select the operating point. */
typedef struct hq_params {
    int32_t tile;        /* elements per RHT tile; must be 128 */
    int32_t lattice;     /* enum hq_lattice */
    float alpha;         /* scale: u = H_128 D x * alpha / sqrt(128) (or (Q x) * alpha); finite, > 0 */
    int32_t rice_k;      /* Rice parameter, 0..15 */
    uint64_t seed;       /* seeds the sign diagonal D and the dither */
    int32_t dither;      /* 0: none; 1: subtractive dither (page section 4; the KV path) */
    int32_t chunk_tiles; /* tiles per chunk; must be 32 */
    const float *rotation; /* KV caches only (hq_kv_init, hq_rate_kv, hq_calibrate_kv); NULL elsewhere.
                            * NULL: the sign diagonal D and H_128 (the default).  Otherwise device
                            * memory, 16-byte aligned: a 128 x 128 orthogonal fp32 matrix Q,
                            * row-major, used in place of H_128 D / sqrt(128):
                            *   u_i = (sum_j Q[i][j] x_j) * alpha,
                            *   x_hat_j = sum_i Q[i][j] ((point - d)_i * fp32(1 / alpha)),
                            * each sum one fp32 fma per term in increasing index from +0.  Must
                            * stay valid and unchanged while the cache is in use.  The weights
                            * entry points return HQ_EUNSUPPORTED when it is set. */
    int32_t rice_dk_last;  /* 0..15.  Bit-stripping halves the last symbol of each A2, D4 or E8 block
                            * (b', q3', m7'), so its best Rice parameter is smaller: it is coded with
                            * max(rice_k - rice_dk_last, 0), every other symbol with rice_k (Z: all
                            * with rice_k).  0: one parameter for all symbols.  The remainder plane
                            * then holds each symbol's k_i low bits at the running sum of the k_i. */
    int32_t reserved;      /* 0 */
} hq_params;               /* 48 bytes */

/* Device-resident statistics written by the kernels (zeroed by each call
 * that takes it).  40 bytes, 8-byte aligned.
 *
 * The integer range of the codes: the pages map lattice points to an integer
 * embedding that is meant to fit 8-bit storage, with alpha calibrated so that
 * the codes do not overflow it (HyperQuant explainer pages, "Methodology" 2,
 * the integer implementation).  The Rice code itself is unbounded, so nothing
 * is clamped; the encoder reports how the call's codes sit against int8:
 *   max_abs_code        the largest |q_i| over every code coordinate q_i of the
 *                       call (the embedding's integers before bit-stripping:
 *                       Z q; A2 (a, b); D4 q; E8 the 2E8 coordinates 2 m + c);
 *   int8_overflow_count the number of code coordinates outside [-128, 127].
 * The encoders (hq_quantize, hq_quantize_static, hq_kv_append) and the rate
 * passes (hq_rate, hq_rate_kv, hq_calibrate*) report both; a KV cache's running
 * stats keep the maximum and the sum over its appends.  Decoding leaves them 0. */
typedef struct hq_stats {
    uint32_t status;       /* HQ_ST_* bits */
    uint32_t max_symbol;   /* bitwise OR of all zigzag symbols coded: its bit length bounds them */
    uint64_t payload_bits; /* sum of Rice codeword lengths plus E8 coset bits */
    uint64_t stream_words; /* words the stream needs (= offsets[n_chunks] when it fit) */
    uint32_t max_abs_code; /* max |code coordinate| (above) */
    uint32_t reserved;     /* 0 */
    uint64_t int8_overflow_count; /* code coordinates outside [-128, 127] (above) */
} hq_stats;

/* One row of a KV cache's append table (device memory; written by
 * hq_kv_append's kernel).  32 bytes. */
typedef struct hq_kv_append_row {
    uint64_t first_chunk; /* global index of the append's first chunk */
    int64_t token0;       /* first token of the append */
    int32_t tokens;       /* T */
    float alpha;          /* alpha used for this append */
    float scale_fwd;      /* fp32(alpha / sqrt(128)); alpha with a dense rotation */
    float scale_inv;      /* fp32(1 / (alpha * sqrt(128))); fp32(1 / alpha) with a dense rotation */
} hq_kv_append_row;

/* A compressed KV cache for one of K or V of one layer (page section 4: KV
 * bias correction with a +-1 sign rotation and subtractive dither).  Plain
 * data: device buffers owned by the caller, and host-side counters that
 * hq_kv_append advances.  One K and one V cache are two of these. */
typedef struct hq_kv_cache {
    uint32_t *d_words;          /* stream, cap_words words */
    uint64_t cap_words;
    uint64_t *d_offsets;        /* chunk offsets, offsets_cap entries (>= total chunks + 1) */
    uint64_t offsets_cap;
    hq_kv_append_row *d_table;  /* one row per append, table_cap rows */
    uint64_t table_cap;
    uint64_t *d_tail;           /* two words: the append numbered a reads the next free stream word from
                                   d_tail[a & 1] and writes the new end to d_tail[(a + 1) & 1] */
    hq_stats *d_stats;          /* accumulated over appends (not zeroed by hq_kv_append) */
    int32_t heads;              /* H */
    int32_t head_dim;           /* must be 128 */
    hq_params params;           /* lattice, k, seed, dither for every append */
    int64_t tokens;             /* host: tokens appended so far */
    uint64_t chunks;            /* host: chunks appended so far */
    uint64_t appends;           /* host: appends so far */
} hq_kv_cache;

/* --------------------------------------------------------------------- sizes */

/* Number of chunks of an R x C weight matrix and an upper bound on its stream
 * size in words for symbols of magnitude at most max_abs_symbol (pass 0 for
 * 255): per chunk, coset + remainder words plus one unary bit per symbol plus
 * (2 max_abs_symbol + 1) >> k zeros per symbol, rounded up to words.  A call
 * whose symbols exceed the assumption reports HQ_ST_CAPACITY instead of
 * overrunning.  Host only; returns HQ_OK or HQ_EINVAL. */
HQ_API int hq_stream_bound(int64_t rows, int64_t cols, const hq_params *p, uint32_t max_abs_symbol,
                    uint64_t *max_words, uint64_t *n_chunks);

/* Bytes of device workspace hq_quantize / hq_kv_append need for n_chunks
 * chunks (8 bytes of chunk look-back state per chunk, a chunk ticket, a CTA
 * counter and the call's stats accumulator), rounded up to 256.  Host only. */
HQ_API int hq_workspace_bytes(uint64_t n_chunks, size_t *bytes);

/* ------------------------------------------------------------ weights path */

/* Quantize and encode an R x C bf16 matrix (page sections 1-3; section 4's
 * dither too if p->dither).
 *   x         device, bf16, element (r, c) at x[r * ld + c]; ld >= cols, ld % 8 == 0.
 *   d_stream  device, cap_words uint32 words, written [0, stream_words).
 *   d_offsets device, n_chunks + 1 uint64 entries, all written.
 *   d_stats   device hq_stats or NULL; replaced by this call's stats, written by
 *             the kernel when it finishes.
 *   workspace device, >= hq_workspace_bytes(n_chunks); overwritten (contents
 *             need no initialisation; the call clears what it uses).
 * Sign index of element (r, c) is c; dither counter (if any) is r * cols + c.
 * Rows * cols may be 0 (then only offsets[0] = 0 and stats are written). */
HQ_API int hq_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, uint32_t *d_stream,
                uint64_t cap_words, uint64_t *d_offsets, hq_stats *d_stats, void *workspace, size_t ws_bytes,
                void *cuda_stream);

/* Decode and dequantize a stream made by hq_quantize with the same rows,
 * cols and params (page sections 1-3 inverted).
 *   d_stream   device, stream_words words (offsets are checked against it).
 *   d_offsets  device, n_chunks + 1 entries.
 *   out        device; out_dtype 0: bf16 (round to nearest even), 1: fp32
 *              (the value before bf16 rounding); element (r, c) at out[r * ld + c],
 *              ld >= cols, ld % 8 == 0 (bf16) or ld % 4 == 0 (fp32).
 *   d_stats    device or NULL; zeroed, then HQ_ST_CORRUPT is set for a bad chunk
 *              (whose tiles are written as zeros). */
HQ_API int hq_dequantize(const uint32_t *d_stream, uint64_t stream_words, const uint64_t *d_offsets, int64_t rows,
                  int64_t cols, const hq_params *p, void *out, int out_dtype, int64_t ld, hq_stats *d_stats,
                  void *cuda_stream);

/* A set of equally shaped matrices in one launch (a strided batch), for coding a
 * model's weight set in bulk.  Item i of `batch`:
 *   input    x + i * x_stride (elements; x_stride % 8 == 0 and >= (rows - 1) * ld + cols),
 *   stream   d_stream + i * stream_stride (words; stream_stride >= cap_words, cap_words
 *            each; any stride: the items' streams need no alignment of their own),
 *   offsets  d_offsets + i * (n_chunks + 1),
 *   stats    d_stats + i (or d_stats NULL).
 * Each item's stream, offsets and stats are exactly what hq_quantize of that matrix alone
 * would write; one launch codes all of them, which removes the start-up and the partly
 * idle last wave that each separate launch has.  workspace >= hq_batch_workspace_bytes
 * (batch, n_chunks) with n_chunks the chunks of one matrix.  batch 0 writes nothing;
 * batch 1 is hq_quantize.  HQ_EUNSUPPORTED when batch * n_chunks reaches 2^31.  Errors
 * otherwise as hq_quantize; asynchronous on cuda_stream.  No counterpart in the paper:
 * the pages code each tensor on its own, and the batch only changes how the work is
 * launched. */
HQ_API int hq_batch_workspace_bytes(int64_t batch, uint64_t n_chunks, size_t *bytes);
HQ_API int hq_quantize_batch(const void *x, int64_t batch, int64_t x_stride, int64_t rows, int64_t cols, int64_t ld,
                             const hq_params *p, uint32_t *d_stream, uint64_t stream_stride, uint64_t cap_words,
                             uint64_t *d_offsets, hq_stats *d_stats, void *workspace, size_t ws_bytes,
                             void *cuda_stream);

/* The inverse of hq_quantize_batch: item i's stream (stream_words words, checked against
 * its offsets) at d_stream + i * stream_stride, offsets at d_offsets + i * (n_chunks + 1),
 * output at out + i * out_stride elements (out_stride % 8 == 0 for bf16, % 4 for fp32,
 * >= (rows - 1) * ld + cols), stats d_stats + i (HQ_ST_CORRUPT per item).  Each item's
 * output is exactly hq_dequantize's.  batch 1 is hq_dequantize.  HQ_EUNSUPPORTED when
 * batch * n_chunks exceeds 2^27. */
HQ_API int hq_dequantize_batch(const uint32_t *d_stream, uint64_t stream_stride, uint64_t stream_words,
                               const uint64_t *d_offsets, int64_t batch, int64_t rows, int64_t cols,
                               const hq_params *p, void *out, int out_dtype, int64_t ld, int64_t out_stride,
                               hq_stats *d_stats, void *cuda_stream);

/* Decode fused into its consumer: y = W x for a compressed matrix W, without
 * writing W to memory.  The pages name the cost of the variable-length format at
 * inference ("Results": decode adds latency on an H100); here each decoded
 * 128-element tile goes straight into a dot product, so W is read at its
 * compressed size (about R/8 bytes per element) instead of 2 bytes of bf16.
 *   W      : the stream of hq_quantize (d_stream, stream_words, d_offsets, rows,
 *            cols, p as for hq_dequantize); its elements are taken exactly as
 *            hq_dequantize stores them in bf16.
 *   d_x    : device, bf16 [cols], 16-byte aligned.
 *   d_y    : device, fp32 [rows]: y[r] = sum_j W[r, j] * x[j], bf16 products
 *            (exact in fp32) accumulated in fp32: per tile a sequential fma over
 *            each lane's 32 elements and a fixed 4-lane tree, then the row's
 *            tiles in column order (results do not depend on scheduling).
 *   workspace, ws_bytes : device, >= hq_gemv_workspace_bytes (one float per
 *            tile), 16-byte aligned.
 * d_stats as hq_dequantize (HQ_ST_CORRUPT; a corrupt chunk's tiles count as 0).
 * Asynchronous on cuda_stream; errors as hq_dequantize. */
HQ_API int hq_gemv_workspace_bytes(int64_t rows, int64_t cols, size_t *bytes);
HQ_API int hq_gemv(const uint32_t *d_stream, uint64_t stream_words, const uint64_t *d_offsets, int64_t rows,
                   int64_t cols, const hq_params *p, const void *d_x, float *d_y, void *workspace, size_t ws_bytes,
                   hq_stats *d_stats, void *cuda_stream);

/* No counterpart in the paper: an addition for callers that cannot allocate.
 *
 * hq_quantize without a workspace, for callers that hold only their input and
 * output buffers and may not allocate device memory: for example a plug-in
 * running inside a host application that owns every device allocation, or
 * code on a path where cudaMalloc (which can synchronise the device) is not
 * allowed.  Arguments, results and status are those of hq_quantize; the
 * caller still passes x, d_stream, d_offsets and (optionally) d_stats.
 *
 * The encoder's scratch (8 bytes of chunk look-back state per chunk, a ticket
 * and a counter word, and a stats accumulator) lives in a fixed array of HQ_STATIC_SCRATCH_BYTES inside
 * libhq.so's device image; every GPU that loads the library holds it until the
 * process exits.  Limit: at most HQ_STATIC_MAX_CHUNKS chunks (4096 elements
 * each, about 537 million elements); a larger matrix returns HQ_EUNSUPPORTED
 * and enqueues nothing.
 *
 * Every call looks up the array's device address in the current context
 * (cudaGetSymbolAddress, with the caller's device current), so a call made
 * after cudaDeviceReset, or from another context, finds the array where that
 * context has it.  The first call in a context may load the library's device
 * code (lazy module loading): make that first call before any stream capture.
 * All calls share the one array and each clears the part it uses with a
 * cudaMemsetAsync on its own stream, so calls that overlap on the GPU (other
 * streams, or other host threads, without ordering between them) race and
 * corrupt each other's streams: serialise them.  The call allocates nothing:
 * no cudaMalloc, cudaFree or allocating library routine. */
#define HQ_STATIC_SCRATCH_BYTES (1u << 20)
#define HQ_STATIC_MAX_CHUNKS 131066u
HQ_API int hq_quantize_static(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p,
                              uint32_t *d_stream, uint64_t cap_words, uint64_t *d_offsets, hq_stats *d_stats,
                              void *cuda_stream);

/* ------------------------------------------------------------- several GPUs */

/* Add base to count chunk offsets (device uint64, 8-byte aligned), in place.
 * The coding path shards into independent tensors with no exchange: each GPU
 * codes its share into its own streams and offsets.  To read the shards as one
 * global stream, each GPU moves its offsets by the global word index at which
 * its part starts (the sum of the word counts of the GPUs before it, one gather
 * of 8 bytes per GPU).  The pages describe a single-device method; this is the
 * only step that several GPUs add.  count 0 is a no-op.  HQ_EINVAL for a null or
 * misaligned pointer; asynchronous on cuda_stream. */
HQ_API int hq_offsets_add(uint64_t *d_offsets, uint64_t count, uint64_t base, void *cuda_stream);

/* ----------------------------------------------------------------- rate targeting */

/* The rate of a quantize call, without its stream.  The pages state that alpha
 * is calibrated and that the realized rate lands within about 0.01 bit per
 * scalar of any target (HyperQuant explainer pages, "Methodology" 2 and 3).
 * This runs the quantize path up to the Rice code lengths and adds into *d_stats
 * (zeroed first, on cuda_stream) exactly what hq_quantize with the same
 * arguments reports:
 *   payload_bits  Rice codeword bits plus E8 coset bits (HQ_ST_RANGE clear);
 *   stream_words  the words hq_quantize would write (coset, remainder and unary
 *                 planes of every chunk), an exact capacity for it;
 *   max_symbol    the OR of all symbols; status  HQ_ST_RANGE as in hq_quantize.
 * x, rows, cols, ld, p and errors are those of hq_quantize; nothing else is
 * written and no workspace is needed.  Asynchronous on cuda_stream. */
HQ_API int hq_rate(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p, hq_stats *d_stats,
                   void *cuda_stream);

/* hq_rate for a block of KV tokens: kv is bf16 [heads, T, 128] with token stride
 * ld_token and head stride ld_head (elements), the tokens being positions
 * tok0 .. tok0 + T - 1 of the cache (their dither counters).  The rate equals
 * that of hq_kv_append of the same tokens at that position, in any split into
 * appends.  HQ_EINVAL for heads <= 0, T < 0, tok0 < 0 or a bad pointer/stride. */
HQ_API int hq_rate_kv(const void *kv, int32_t heads, int64_t T, int64_t ld_token, int64_t ld_head, int64_t tok0,
                      const hq_params *p, hq_stats *d_stats, void *cuda_stream);

/* What to calibrate: payload bits per scalar to reach, its tolerance, the alpha
 * bracket and the Rice parameters to try. */
typedef struct hq_calib_spec {
    double target_bps;           /* > 0 */
    double tol;                  /* >= 0; stop when |rate - target| <= tol (e.g. 0.002) */
    double alpha_lo, alpha_hi;   /* 0 < lo < hi; the bracket (e.g. 1e-3, 1e4) */
    int32_t k_lo, k_hi;          /* 0 <= k_lo <= k_hi <= 15 */
    int32_t max_iter;            /* bisection steps per k, 0..200 (e.g. 60) */
    int32_t reserved;            /* 0 */
} hq_calib_spec;                 /* 48 bytes */

typedef struct hq_calib_result {
    float alpha;                 /* the calibrated alpha (fp32, as hq_params holds it) */
    int32_t k;                   /* the chosen Rice parameter, -1 if none */
    double bps;                  /* payload bits per scalar at (alpha, k) */
    int32_t evaluations;         /* rate passes run */
    uint32_t status;             /* OR of the HQ_ST_* bits the passes saw */
} hq_calib_result;               /* 24 bytes */

/* Choose alpha (and k) on the device so that the payload rate of quantizing x
 * meets a target.  For each k in [k_lo, k_hi], if rate(alpha_lo) <= target <=
 * rate(alpha_hi), alpha is bisected at the geometric mid point sqrt(lo * hi)
 * (evaluated at its fp32 rounding) until |rate - target| <= tol, at most
 * max_iter steps; without convergence the result is the mid point of the final
 * bracket.  The k with the largest alpha (the finest lattice at that rate)
 * wins, the first on ties.  rate = hq_rate's payload_bits / (rows * cols); a
 * pass that flags HQ_ST_RANGE counts as +infinity.
 *
 * p gives the lattice, seed and dither (its alpha and rice_k are ignored);
 * d_stats is device scratch.  Unlike every other entry point this one
 * SYNCHRONISES: each pass is copied back and waited for on cuda_stream, and the
 * result is in *out when the call returns.  Returns HQ_OK; HQ_EUNSUPPORTED if
 * no k brackets the target (out->k = -1); HQ_EINVAL for a bad spec, pointer or
 * empty matrix; HQ_ECUDA on a CUDA error. */
HQ_API int hq_calibrate(const void *x, int64_t rows, int64_t cols, int64_t ld, const hq_params *p,
                        const hq_calib_spec *spec, hq_stats *d_stats, void *cuda_stream, hq_calib_result *out);

/* hq_calibrate for KV tokens (layout as hq_rate_kv); rate = payload bits /
 * (heads * T * 128). */
HQ_API int hq_calibrate_kv(const void *kv, int32_t heads, int64_t T, int64_t ld_token, int64_t ld_head,
                           int64_t tok0, const hq_params *p, const hq_calib_spec *spec, hq_stats *d_stats,
                           void *cuda_stream, hq_calib_result *out);

/* ----------------------------------------------------------------- KV path */

/* Fill a hq_kv_cache with the caller's buffers and zero its two tail words
 * and its stats (two small cudaMemsetAsync on cuda_stream).  p->dither is
 * normally 1; p->alpha is unused (each append gives its own).  p->rotation, if
 * set, rotates every append, read and score of this cache (the table rows then
 * hold scale_fwd = alpha and scale_inv = fp32(1 / alpha)). */
HQ_API int hq_kv_init(hq_kv_cache *cache, int32_t heads, int32_t head_dim, const hq_params *p, uint32_t *d_words,
               uint64_t cap_words, uint64_t *d_offsets, uint64_t offsets_cap, hq_kv_append_row *d_table,
               uint64_t table_cap, uint64_t *d_tail, hq_stats *d_stats, void *cuda_stream);

/* Append T tokens to a compressed KV cache: the KV-cache quantizer of the pages
 * (HyperQuant explainer pages, "Methodology" 4, KV bias correction: a
 * per-layer rotation, here the seeded sign diagonal with H_128 or the cache's
 * dense rotation, then the lattice quantizer with subtractive dither; sections
 * 1-3 for the RHT, the lattice and the Rice code; arXiv abstract, step (iv)).
 * kv is device bf16 [H, T, 128], element (h, t, d) at
 * kv[h * ld_head + t * ld_token + d] (both strides % 8 == 0).  The chunks are
 * written from the cache's device-resident tail on, so appends queue without a
 * host sync.  Dither counter of (token, head, dim) is (token * H + head) * 128
 * + dim, token counted from the cache start; sign index is dim.  alpha is this
 * append's scale (stored in its table row).  Advances cache->tokens, chunks,
 * appends on the host.  workspace: >= hq_workspace_bytes(H * ceil(T / 32)). */
HQ_API int hq_kv_append(hq_kv_cache *cache, const void *kv, int64_t T, int64_t ld_token, int64_t ld_head, float alpha,
                 void *workspace, size_t ws_bytes, void *cuda_stream);

/* Read a compressed KV cache back: the exact inverse of every append (the same
 * pages and sections as hq_kv_append: Rice decode, re-inserted membership bits,
 * the dither subtracted, unscaled, the inverse rotation).  Decode the first len
 * tokens of every head: out [H, len, 128], element
 * (h, t, d) at out[h * out_ld_head + t * out_ld_token + d]; out_dtype as in
 * hq_dequantize.  len <= cache->tokens. */
HQ_API int hq_kv_read(const hq_kv_cache *cache, void *out, int out_dtype, int64_t len, int64_t out_ld_token,
               int64_t out_ld_head, void *cuda_stream);

/* Attention scores over a compressed K cache, without writing K to memory:
 * scores[(h * group + g) * scores_ld + t] = sum_d K[h, t, d] * q[h * group + g, d]
 * for every KV head h, query head g of its group and token t < len; K[h, t, :]
 * is exactly the bf16 row hq_kv_read stores (after un-dithering), products are
 * exact in fp32 and accumulated as in hq_gemv.
 *   d_q       : device, bf16 [heads * group, 128], 16-byte aligned.
 *   group     : query heads per KV head (grouped-query attention), >= 1.
 *   d_scores  : device, fp32 [heads * group, scores_ld], scores_ld >= len;
 *               columns >= len are not written.
 * Status bits go to the cache's d_stats as for hq_kv_read.  Asynchronous. */
HQ_API int hq_kv_scores(const hq_kv_cache *cache, const void *d_q, int32_t group, float *d_scores, int64_t len,
                        int64_t scores_ld, void *cuda_stream);

/* Draw a Haar-uniform rotation for hq_params.rotation: d_q (device, 16-byte
 * aligned, 128 x 128 fp32 row-major) = the orthogonal factor Q of G = Q R with R
 * upper triangular and positive on its diagonal, where G[i][j] is the standard
 * normal draw e = 128 i + j: h = splitmix64(seed ^ 0x524F544E, e), u1 = (h >> 32
 * + 1/2) 2^-32, u2 = (h & 0xFFFFFFFF) 2^-32, g = sqrt(-2 ln u1) cos(2 pi u2).  That
 * factor is Haar-distributed on O(128) (Mezzadri 2007).  Computed in double on one
 * CTA (modified Gram-Schmidt) and rounded once to fp32; another QR method gives the
 * same fp32 matrix to within one unit in the last place.  One call per cache
 * (per layer and K/V, each with its own seed); asynchronous on cuda_stream.
 * HQ_EINVAL for a null or misaligned d_q. */
HQ_API int hq_haar_rotation(uint64_t seed, float *d_q, void *cuda_stream);

/* ---------------------------------------------------------------- misc */

/* Human-readable text for a return code (negative) or status bit mask (>= 0). */
HQ_API const char *hq_status_string(int code);

/* HQ_OK if the current CUDA device is sm_100 (B200-class) and the library's
 * kernels can run on it; HQ_EUNSUPPORTED or HQ_ECUDA otherwise. */
HQ_API int hq_device_check(void);

/* Testing aid: the number of polls a chunk's look-back makes on a
 * predecessor that has not published before it gives up and sets
 * HQ_ST_TIMEOUT (0 restores the default, 2^22).  Process-wide; affects calls
 * made after it.  A timed-out call's stream is unspecified but every write
 * stays inside [0, cap_words). */
HQ_API void hq_debug_set_spin_limit(uint32_t polls);

/* Testing aid: which form of the quantize kernel runs.  0 (default) chooses by
 * size: launches of at most 32 chunks (16 with a dense rotation, except one-token
 * appends) run in one CTA (no workspace is touched: the fewest steps for a KV
 * append of a few tokens; a one-token append gives each chunk to a half-warp), of
 * at most 2 chunks per SM the wide form (16 warps share a chunk, 16 lanes per
 * tile), of at most three quarters of the per-warp form's resident warps (all of
 * them with dither; 1776 and 2368 chunks on a B200) the grouped form (4 warps
 * share a chunk), larger ones the per-warp form (a warp encodes whole chunks: the
 * highest throughput).  1 forces per-warp, 2 grouped, 3 wide,
 * 4 the single CTA (per-warp beyond its limit).  A dense rotation uses the grouped
 * form unless the single CTA applies; a second Rice parameter replaces the wide
 * form by the grouped one.  All give identical streams, offsets and stats.
 * Process-wide; HQ_EINVAL outside 0..4. */
HQ_API int hq_debug_set_encode_path(int path);

/* Testing aid: the nearest point of the lattice in its integer embedding
 * (the decoder the quantize kernels run; HyperQuant explainer pages,
 * "Methodology" 2) for n_blocks vectors.
 *   d_v : device, n_blocks x dim fp32 values (dim = 1, 2, 4, 8 for Z, A2, D4,
 *         E8), 4-byte aligned, read only.
 *   d_q : device, n_blocks x dim int32 codes out (E8: 2E8 = 2D8 u (2D8 + 1);
 *         D4: sum even; A2: (a, b) with a = b mod 2; Z: the rounded value).
 * Asynchronous on cuda_stream.  HQ_EINVAL for a bad lattice, a negative count
 * or a null / misaligned pointer; HQ_ECUDA if the launch fails. */
HQ_API int hq_debug_nearest(int lattice, const float *d_v, int64_t n_blocks, int32_t *d_q, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
