// hq_encode.cuh -- quantize + encode kernels (HyperQuant "Methodology" sections
// 1-4): per 128-element tile, seeded sign flip, FWHT-128, scale, optional
// subtractive dither, nearest lattice point, bit-stripping, zigzag, Rice planes;
// and the rate-only pass that counts the same codes without writing them.
//
// Four forms with identical output, chosen by launch size (hq_encode.cu):
//  * per-warp (throughput; more than 1776 chunks on a B200, 2368 with dither):
//    one warp encodes one chunk
//    (32 tiles) in 4 rounds of 8 tiles; four lanes share a tile, 32 elements
//    each, loaded as 64 contiguous bytes per lane with cp.async one round ahead;
//    the transform runs in registers (16 float2 per lane, packed fp32 adds, the
//    last two butterfly stages across lanes by shuffle); each lane decodes its
//    32/N lattice blocks into 32 zigzag symbols; a warp scan of unary lengths
//    places every codeword in a per-warp shared stage holding the chunk;
//  * grouped (latency; up to 1776 chunks, 2368 with dither): four warps share
//    a chunk, one round each, meeting at a named barrier per chunk;
//  * wide (lowest latency; up to 296 chunks): sixteen warps share a chunk,
//    sixteen lanes per tile, one 8-element block per lane;
//  * single CTA (up to 32 chunks, such as a KV append of a few tokens): the
//    CTA's warps encode the chunks into their own stages and one warp scans
//    the sizes into offsets, with no workspace, ticket or look-back; for a
//    one-token append (one-tile chunks) each half-warp takes a chunk in the
//    wide form's layout.
// In the first three a persistent grid takes chunk tickets from a global
// counter, so a chunk's predecessors are always already running, and a
// single-pass decoupled look-back over 64-bit (flag, value) words gives each
// chunk's word offset (bounded waits: HQ_ST_TIMEOUT).  A chunk publishes its
// size as soon as it is encoded and resolves its offset one chunk later, when
// its predecessors have normally published; its stage is then copied out
// coalesced.  A chunk larger than the stage is re-encoded by a path that sets
// its bits in place in global memory (the same bits; only for extreme codes).
// Options: the dense KV rotation in place of the sign diagonal and H_128 (ROT;
// grouped and single-CTA forms), a second Rice parameter for the last symbol of
// each lattice block (MIXED; all forms but the wide one).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_device.cuh"

namespace hq {

namespace {

constexpr unsigned long long kFlagAgg = 1ull << 62;
constexpr unsigned long long kFlagInc = 2ull << 62;
constexpr unsigned long long kValMask = (1ull << 62) - 1;

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Decoupled look-back over 64-bit words (flag in the top two bits, value
// below): 0 = nothing yet, AGG = the chunk's own word count, INC = the chunk's
// inclusive prefix.  A chunk publishes its count as soon as it is encoded and
// resolves its offset later, so waits are short.

// Publish chunk c's word count (the first chunk of a stream, `first`, publishes its
// inclusive prefix: the walk-back of later chunks stops there).
__device__ __forceinline__ void lookback_publish(unsigned long long *lb, unsigned long long c,
                                                 unsigned long long agg, bool first) {
    if ((threadIdx.x & 31) == 0) st_relaxed_u64(lb + c, (first ? kFlagInc : kFlagAgg) | agg);
}

// The look-back word of predecessor c - 1 - lane (INC with value 0 before chunk 0):
// the first window of a resolve, loaded early so its latency overlaps other work.
__device__ __forceinline__ unsigned long long lookback_peek(const unsigned long long *lb, unsigned long long c) {
    const long long idx = (long long)c - 1 - (threadIdx.x & 31);
    return (idx >= 0) ? ld_relaxed_u64(lb + idx) : kFlagInc;
}

// Exclusive prefix (in words) of chunk c: walk back over predecessors 32 at a
// time until one with an inclusive prefix, summing counts; then publish c's
// inclusive prefix.  `first` is lookback_peek(lb, c), taken earlier.  Whole warp
// calls it.  Bounded: gives up after spin_limit polls.
__device__ __noinline__ unsigned long long lookback_resolve(unsigned long long *lb, unsigned long long c,
                                                            unsigned long long agg, uint32_t spin_limit,
                                                            bool &timed_out, unsigned long long first,
                                                            bool stream_first) {
    const int lane = threadIdx.x & 31;
    if (stream_first) return 0;
    unsigned long long excl = 0;
    long long pos = (long long)c - 1;
    uint32_t spins = 0;
    bool use_first = true;
    while (true) {
        const long long idx = pos - lane;
        const unsigned long long v = use_first ? first : (idx >= 0) ? ld_relaxed_u64(lb + idx) : kFlagInc;
        use_first = false;
        const unsigned flag = (unsigned)(v >> 62);
        const unsigned inc = __ballot_sync(0xffffffffu, flag == 2u);
        const unsigned zero = __ballot_sync(0xffffffffu, flag == 0u);
        const int first_inc = inc ? __ffs(inc) - 1 : 32;
        const unsigned relevant = (first_inc >= 31) ? 0xffffffffu : ((2u << first_inc) - 1u);
        if (zero & relevant) {
            if (++spins > spin_limit) {
                timed_out = true;
                break;
            }
            __nanosleep(32);
            continue;
        }
        excl += warp_sum_u64(lane <= first_inc ? (v & kValMask) : 0ull);
        if (first_inc < 32) break;
        pos -= 32;
    }
    if (lane == 0) st_relaxed_u64(lb + c, kFlagInc | (excl + agg));
    return excl;
}

// A lane's integer range of the codes it has produced: the largest code key (see
// code_abs_of_key) and the count of code coordinates outside int8, which is taken
// from the symbols only when a round's key reaches key_int8_limit (rare).
struct CodeRange {
    uint32_t key = 0, ovf = 0;
    template <int LAT, int S>
    __device__ __forceinline__ void add(uint32_t rkey, const uint32_t (&z)[S], uint32_t cbits) {
        key = max(key, rkey);
        if (rkey >= key_int8_limit<LAT>()) {
            // the out-of-line recount takes its symbols from memory: copy them there only on this
            // rare path, so that z itself stays in registers every round
            uint32_t zc[S];
#pragma unroll
            for (int i = 0; i < S; i++) zc[i] = z[i];
            ovf += int8_overflow<LAT, S>(zc, cbits);
        }
    }
};

// Stats of an encode call.  Every warp adds its part to the workspace accumulator
// (the warp's payload is lane 0's; the accumulator is cleared with the look-back
// words, so the caller's stats need no separate clearing); the last CTA to finish moves the totals to the caller's stats,
// replacing them (hq_quantize) or adding to them (a KV cache's running stats).
template <int LAT>
__device__ __forceinline__ void stats_add_warp(const EncodeArgs &a, uint32_t status, uint32_t zor_all,
                                               unsigned long long payload, const CodeRange &rng,
                                               unsigned long long item = 0) {
    status = __reduce_or_sync(0xffffffffu, status);
    zor_all = __reduce_or_sync(0xffffffffu, zor_all);
    const uint32_t key = __reduce_max_sync(0xffffffffu, rng.key);
    const uint32_t ovf = __reduce_add_sync(0xffffffffu, rng.ovf);
    if ((threadIdx.x & 31) == 0) {
        hq_stats *acc = a.acc + item;
        if (status) atomicOr(&acc->status, status);
        if (zor_all) atomicOr(&acc->max_symbol, zor_all);
        if (payload) atomicAdd((unsigned long long *)&acc->payload_bits, payload);
        if (key) atomicMax(&acc->max_abs_code, code_abs_of_key<LAT>(key));
        if (ovf) atomicAdd((unsigned long long *)&acc->int8_overflow_count, (unsigned long long)ovf);
    }
}

// Whole CTA calls it once, at its end.  The last CTA moves every item's accumulator.
__device__ __forceinline__ void stats_finish_cta(const EncodeArgs &a) {
    __syncthreads();
    if (threadIdx.x != 0) return;
    __threadfence();
    if (atomicAdd(a.done, 1u) != gridDim.x - 1) return;
    __threadfence();
    if (!a.stats) return;
    const unsigned long long items = a.batch > 1 ? a.batch : 1ull;
    for (unsigned long long i = 0; i < items; i++) {
        const hq_stats *acc = a.acc + i;
        hq_stats *out = a.stats + i;
        const uint32_t st = ld_relaxed_u32(&acc->status), mx = ld_relaxed_u32(&acc->max_symbol);
        const unsigned long long pb = ld_relaxed_u64((const unsigned long long *)&acc->payload_bits);
        const unsigned long long sw = ld_relaxed_u64((const unsigned long long *)&acc->stream_words);
        const uint32_t am = ld_relaxed_u32(&acc->max_abs_code);
        const unsigned long long ov = ld_relaxed_u64((const unsigned long long *)&acc->int8_overflow_count);
        if (a.stats_add) {
            if (st) atomicOr(&out->status, st);
            if (mx) atomicOr(&out->max_symbol, mx);
            if (pb) atomicAdd((unsigned long long *)&out->payload_bits, pb);
            if (am) atomicMax(&out->max_abs_code, am);
            if (ov) atomicAdd((unsigned long long *)&out->int8_overflow_count, ov);
        } else {
            out->status = st;
            out->max_symbol = mx;
            out->payload_bits = pb;
            out->max_abs_code = am;
            out->reserved = 0u;
            out->int8_overflow_count = ov;
        }
        out->stream_words = sw;
    }
}

// The item of a strided batch that chunk c belongs to, and c's index within it.
struct ItemChunk {
    unsigned long long item, local;
};
// NARROW: the launch has fewer than 2^27 chunks (32-bit divisions suffice).
template <bool NARROW = false>
__device__ __forceinline__ ItemChunk item_chunk(const EncodeArgs &a, unsigned long long c) {
    ItemChunk r{0ull, c};
    if (a.batch > 1) {
        if (NARROW) {
            const uint32_t q = (uint32_t)c / (uint32_t)a.item_chunks;
            r.item = q;
            r.local = (uint32_t)c - q * (uint32_t)a.item_chunks;
        } else {
            divmod_u64(c, a.item_chunks, r.item, r.local);
        }
    }
    return r;
}

// Which tile maps a kernel handles: both (chosen at run time by TileMap::kv), or one known
// at compile time (the other's code compiled out).
constexpr int kMapAny = 0, kMapWeights = 1, kMapKv = 2;

// Where the tiles of one chunk are (computed once per chunk).
struct ChunkGeo {
    int ntiles;
    long long xoff;   // elements from x to this chunk's matrix (a batch item; 0 otherwise)
    // weights: tile ti of the chunk is row row0 + (tc0 + ti) / tpr, tile column (tc0 + ti) % tpr
    long long row0;
    int tc0, tpr;
    // kv: head h, tokens tok_base + ti
    long long h, tok_base;

    // MAP: kMapAny, or the map the caller knows it has (kMapWeights, kMapKv);
    // NARROW: c < 2^27, so the chunk's first tile 32 c fits 32 bits
    template <int MAP = kMapAny, bool NARROW = false>
    __device__ __forceinline__ void init(const TileMap &m, unsigned long long c) {
        xoff = 0;
        if (MAP == kMapKv || (MAP == kMapAny && m.kv)) {
            const long long cph = (m.tokens + 31) / 32;
            unsigned long long hq_, rq;
            divmod_u64(c, (unsigned long long)cph, hq_, rq);
            h = (long long)hq_;
            tok_base = (long long)rq * 32;
            long long left = m.tokens - tok_base;
            ntiles = (int)(left < 32 ? left : 32);
        } else {
            tpr = (int)(m.cols / kTile);
            long long t0 = (long long)c * 32;
            long long all = m.rows * (long long)tpr;
            ntiles = (int)((all - t0) < 32 ? (all - t0) : 32);
            if (NARROW) {
                const uint32_t rq = (uint32_t)t0 / (uint32_t)tpr;
                row0 = rq;
                tc0 = (int)((uint32_t)t0 - rq * (uint32_t)tpr);
            } else {
                unsigned long long rq, cq;
                divmod_u64((unsigned long long)t0, (unsigned long long)tpr, rq, cq);
                row0 = (long long)rq;
                tc0 = (int)cq;
            }
        }
    }
    // Tile ti (< 32) of the chunk: first element, sign-table column, dither counter of its element 0.
    template <int MAP = kMapAny>
    __device__ __forceinline__ bool tile(const TileMap &m, const uint16_t *x, int ti, const uint16_t *&src,
                                         int &tcol, unsigned long long &e0) const {
        if (ti >= ntiles) return false;
        if (MAP == kMapKv || (MAP == kMapAny && m.kv)) {
            long long tok = tok_base + ti;
            src = x + h * m.ld_head + tok * m.ld_tok;
            tcol = 0;
            e0 = (unsigned long long)(((m.tok0 + tok) * m.heads + h) * kTile);
            return true;
        }
        int tc = tc0 + ti;
        long long r = row0;
        if (tc >= tpr) {
            int d = tc / tpr;
            r += d;
            tc -= d * tpr;
        }
        src = x + xoff + r * m.ld + (long long)tc * kTile;
        tcol = tc;
        e0 = (unsigned long long)(r * m.cols + (long long)tc * kTile);
        return true;
    }
};

// Input of one round for one lane: its quarter (32 bf16 = 64 bytes) of tile
// 8r + lane/4.  The bytes are copied ahead of use with cp.async into the
// lane's own 80-byte slot of a per-warp shared buffer (80: 8 consecutive lanes'
// 16-byte accesses hit distinct banks); each lane reads back only what it
// copied, so no warp barrier is needed.
struct RoundInput {
    bool valid;
    int tcol;
    unsigned long long e0;
};

constexpr int kInSlotWords = 20;     // per-lane input slot of the per-warp kernel (80 B)
constexpr int kGroupSlotWords = 36;  // grouped kernel: the slot also parks the 32 symbols (144 B)

template <int MAP = kMapAny>
__device__ __forceinline__ void prefetch_round(const EncodeArgs &a, const ChunkGeo &geo, int r, int lane,
                                               uint32_t *slot) {
    const uint16_t *src = nullptr;
    int tcol;
    unsigned long long e0;
    if (geo.template tile<MAP>(a.map, a.x, r * kTilesPerRound + (lane >> 2), src, tcol, e0)) {
        const uint16_t *g = src + 32 * (lane & 3);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const unsigned sa = (unsigned)__cvta_generic_to_shared(slot + 4 * j);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(g + 8 * j) : "memory");
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Bulk form of the per-warp kernel's input (BULK: weights whose rows hold whole rounds):
// the round's 8 tiles are one 2 KB run of x, copied by a single cp.async.bulk issued by
// lane 0 into the warp's buffer and completed on the warp's mbarrier (transaction count
// 2048 bytes).  Lane l then reads bytes [64 l, 64 l + 64): its quarter l % 4 of tile l / 4,
// as in the per-lane form.
constexpr uint32_t kRoundBytes = kTilesPerRound * kTile * 2;

__device__ __forceinline__ void bulk_prefetch_round(const EncodeArgs &a, const ChunkGeo &geo, int r, uint32_t buf,
                                                    uint32_t mb) {
    const uint16_t *src = nullptr;
    int tcol;
    unsigned long long e0;
    geo.tile<kMapWeights>(a.map, a.x, r * kTilesPerRound, src, tcol, e0);
    // the buffer was last read through the generic proxy (ordered by the caller's __syncwarp)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(kRoundBytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(buf), "l"(src), "r"(kRoundBytes), "r"(mb) : "memory");
}

// Polls of a round's bulk-copy wait before it gives up: at least this many, far above any copy's
// latency (seconds), whatever the look-back's limit (which tests lower to one poll): a CTA must
// not end while a copy into its shared memory is in flight.  (Taken as spin_limit | this, a run-time
// value: a compile-time bound made the kernel about 1 % slower.)
constexpr uint32_t kBulkWaitPolls = 1u << 24;

// Wait for the phase of parity `phase` of mbarrier mb to complete; false after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mb, uint32_t phase, uint32_t limit) {
    for (uint32_t i = 0; i < limit; i++) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done) : "r"(mb), "r"(phase) : "memory");
        if (done) return true;
    }
    return false;
}

template <int MAP = kMapAny>
__device__ __forceinline__ void round_input(const EncodeArgs &a, const ChunkGeo &geo, int r, int lane,
                                            RoundInput &in) {
    const uint16_t *src = nullptr;
    in.tcol = 0;
    in.e0 = 0;
    in.valid = geo.template tile<MAP>(a.map, a.x, r * kTilesPerRound + (lane >> 2), src, in.tcol, in.e0);
}

// The transform of one round for one lane: D x -> H_128 (with the three partner
// lanes), or with ROT the dense rotation Q x (rot_s: its shared form).  Invalid
// tiles transform zeros.  Whole warp (shuffles).
template <bool ROT>
__device__ __forceinline__ void round_transform(const RoundInput &in, const uint4 (&raw)[4], int lane,
                                                const uint32_t *sign_tab, const float *rot_s, float2 (&v)[16]) {
    if constexpr (ROT) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint4 r = in.valid ? raw[j] : make_uint4(0, 0, 0, 0);
            const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int t = 0; t < 4; t++)
                v[4 * j + t] = make_float2(__uint_as_float(wv[t] << 16), __uint_as_float(wv[t] & 0xFFFF0000u));
        }
        rotate_round(v, rot_s, lane);
    } else {
        const uint32_t es = sign_tab[in.tcol * kSignWords + (lane & 3)];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint4 w = in.valid ? raw[j] : make_uint4(0, 0, 0, 0);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int t = 0; t < 4; t++) {
                const uint32_t ww = wv[t] ^ sign_pair_mask(es, 4 * j + t);
                v[4 * j + t] = make_float2(__uint_as_float(ww << 16), __uint_as_float(ww & 0xFFFF0000u));
            }
        }
        fwht128_quarter(v, lane);
    }
}

// One round for one lane: the transform -> * c -> [+ d] -> lattice blocks -> 32
// zigzag symbols, the E8 coset bits of its blocks and the largest code key of the
// round (0 for an invalid tile).  Whole warp must call it.
template <int LAT, bool DITHER, bool ROT = false>
__device__ __forceinline__ void round_symbols(const EncodeArgs &a, const RoundInput &in, const uint4 (&raw)[4],
                                              int lane, const uint32_t *sign_tab, uint32_t (&z)[32],
                                              uint32_t &cbits, uint32_t &rkey, const float *rot_s = nullptr) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    const int q = lane & 3;
    float2 v[16];
    round_transform<ROT>(in, raw, lane, sign_tab, rot_s, v);
    const float2 c2 = make_float2(a.c_scale, a.c_scale);
#pragma unroll
    for (int j = 0; j < 16; j++) v[j] = f2_mul(v[j], c2);

    cbits = 0;
    rkey = 0;
    const unsigned long long eq = in.e0 + 32ull * q;
#pragma unroll
    for (int b = 0; b < 32 / N; b++) {
        float blk[N];
#pragma unroll
        for (int i = 0; i < N; i++) {
            const int e = b * N + i;
            blk[i] = (e & 1) ? v[e >> 1].y : v[e >> 1].x;
        }
        if (DITHER) {
            float d[N];
            dither_block<LAT>(a.seed, eq + (unsigned long long)(b * N), d);
#pragma unroll
            for (int i = 0; i < N; i++) blk[i] = __fadd_rn(blk[i], d[i]);
        }
        uint32_t zz[N];
        cbits |= L::symbols(blk, zz, rkey) << b;
#pragma unroll
        for (int i = 0; i < N; i++) z[b * N + i] = (!DITHER || in.valid) ? zz[i] : 0u;
    }
    if (!in.valid) cbits = 0;
    if (!in.valid) rkey = 0;
}

// N consecutive floats of a lane's shared row (16-byte aligned rows; offsets are
// multiples of N words).
template <int N>
__device__ __forceinline__ void row_load(const uint32_t *r, float (&x)[N]) {
    if (N == 8) {
        const float4 a = reinterpret_cast<const float4 *>(r)[0], b = reinterpret_cast<const float4 *>(r)[1];
        const float t[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < N; i++) x[i] = t[i];
    } else if (N == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(r);
        const float t[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < N; i++) x[i] = t[i];
    } else if (N == 2) {
        const float2 a = *reinterpret_cast<const float2 *>(r);
        x[0] = a.x;
        x[N - 1] = a.y;
    } else {
        x[0] = __uint_as_float(r[0]);
    }
}
template <int N>
__device__ __forceinline__ void row_store(uint32_t *r, const uint32_t (&z)[N]) {
    if (N == 8) {
        reinterpret_cast<uint4 *>(r)[0] = make_uint4(z[0], z[1 % N], z[2 % N], z[3 % N]);
        reinterpret_cast<uint4 *>(r)[1] = make_uint4(z[4 % N], z[5 % N], z[6 % N], z[7 % N]);
    } else if (N == 4) {
        *reinterpret_cast<uint4 *>(r) = make_uint4(z[0], z[1 % N], z[2 % N], z[3 % N]);
    } else if (N == 2) {
        *reinterpret_cast<uint2 *>(r) = make_uint2(z[0], z[N - 1]);
    } else {
        r[0] = z[0];
    }
}

// The same round with the lattice-block loop rolled over a lane-private shared row
// (the 32 transformed values, then their symbols in place): one copy of the block
// code instead of 32/N.  For the latency form, where each warp runs a round once
// and fetching the unrolled code from a cold instruction cache, not issue, bounds
// it.  Leaves the 32 symbols in row[0, 32), their quotient sum and OR, and the largest
// code key of the round (0 for an invalid tile).
template <int LAT, bool DITHER, bool ROT>
__device__ __forceinline__ void round_symbols_rolled(const EncodeArgs &a, const RoundInput &in, const uint4 (&raw)[4],
                                                     int lane, const uint32_t *sign_tab, uint32_t *row,
                                                     uint32_t &cbits, uint32_t &usum, uint32_t &lor,
                                                     uint32_t &rkey, const float *rot_s) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    const int q = lane & 3;
    float2 v[16];
    round_transform<ROT>(in, raw, lane, sign_tab, rot_s, v);
    const float2 c2 = make_float2(a.c_scale, a.c_scale);
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const float2 lo = f2_mul(v[2 * j], c2), hi = f2_mul(v[2 * j + 1], c2);
        reinterpret_cast<float4 *>(row)[j] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    cbits = 0;
    usum = 0;
    lor = 0;
    rkey = 0;
    const int k = a.k, kl = a.k_last;
    const unsigned long long eq = in.e0 + 32ull * q;
#pragma unroll 1
    for (int b = 0; b < 32 / N; b++) {
        float blk[N];
        row_load<N>(row + b * N, blk);
        if (DITHER) {
            float d[N];
            dither_block<LAT>(a.seed, eq + (unsigned long long)(b * N), d);
#pragma unroll
            for (int i = 0; i < N; i++) blk[i] = __fadd_rn(blk[i], d[i]);
        }
        uint32_t zz[N];
        cbits |= L::symbols(blk, zz, rkey) << b;
#pragma unroll
        for (int i = 0; i < N; i++) {
            zz[i] = (!DITHER || in.valid) ? zz[i] : 0u;
            usum += zz[i] >> sym_k<N>(i, k, kl);
            lor |= zz[i];
        }
        row_store<N>(row + b * N, zz);
    }
    if (!in.valid) cbits = 0;
    if (!in.valid) rkey = 0;
}

// Remainder bits of 32 symbols (warp-uniform k) into the lane's k words.
// KSMALL (k <= 4): a group of 8 remainders is built in one register, last
// symbol first (an and and a multiply-add per symbol); otherwise a 64-bit accumulator.
template <bool KSMALL>
__device__ __forceinline__ void put_rem(uint32_t *dst, const uint32_t (&z)[32], int k, bool store) {
    if (k == 0) return;
    if (KSMALL && (k & (k - 1)) == 0) {
        // k in {1, 2, 4}: 32 / k remainders fill a word exactly.  Each symbol's k low bits
        // enter at the top of the word by one funnel shift, (z : acc) >> k, so that when the
        // word is full its first symbol sits in the lowest bits; full words are stored.
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 32; i++) {
            acc = __funnelshift_r(acc, z[i], k);
            if (store) {
                if (i == 7 && k == 4) dst[0] = acc;
                if (i == 15 && k >= 2) dst[k / 2 - 1] = acc;
                if (i == 23 && k == 4) dst[2] = acc;
                if (i == 31) dst[k - 1] = acc;
            }
        }
        return;
    }
    const uint32_t mask = (1u << k) - 1u;
    unsigned long long acc = 0;
    uint32_t nb = 0, w = 0;
#pragma unroll
    for (int g = 0; g < 4; g++) {
        if (KSMALL) {
            const uint32_t pk = 1u << k;
            uint32_t gv = 0;
#pragma unroll
            for (int i = 7; i >= 0; i--) gv = imad(gv, pk, z[8 * g + i] & mask);
            acc |= (unsigned long long)gv << nb;
            nb += 8u * (uint32_t)k;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) {
                acc |= (unsigned long long)(z[8 * g + i] & mask) << nb;
                nb += (uint32_t)k;
                if (nb >= 32u) {
                    if (store) dst[w] = (uint32_t)acc;
                    w++;
                    acc >>= 32;
                    nb -= 32u;
                }
            }
        }
        if (nb >= 32u) {
            if (store) dst[w] = (uint32_t)acc;
            w++;
            acc >>= 32;
            nb -= 32u;
        }
    }
}

// Remainder bits of a lane's 32 symbols with a second Rice parameter kl for the last
// symbol of each lattice block (sym_k): the lane's run starts at bit `lb` of the
// remainder plane, so it shares its first and last words with its neighbours; every
// word is ORed in (the plane is zeroed).  A group of 8 remainders that fits in 32 bits
// is built in one register, last symbol first.
template <int N>
__device__ __forceinline__ void put_rem_mixed(uint32_t *rem, uint32_t lb, const uint32_t (&z)[32], int k, int kl) {
    const uint32_t gbits = group_rem_bits<N>(k, kl);
    if (gbits == 0u) return;
#pragma unroll
    for (int g = 0; g < 4; g++) {
        const uint32_t b0 = lb + (uint32_t)g * gbits;
        if (gbits <= 32u) {
            uint32_t gv = 0;
#pragma unroll
            for (int i = 7; i >= 0; i--) {
                const int ki = sym_k<N>(i, k, kl);
                gv = imad(gv, 1u << ki, z[8 * g + i] & ((1u << ki) - 1u));
            }
            const uint32_t w0 = b0 >> 5, sh = b0 & 31u;
            atomicOr(rem + w0, gv << sh);
            if (sh + gbits > 32u) atomicOr(rem + w0 + 1, gv >> (32u - sh));
        } else {
            uint32_t b = b0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int ki = sym_k<N>(i, k, kl);
                const uint32_t w0 = b >> 5, sh = b & 31u, val = z[8 * g + i] & ((1u << ki) - 1u);
                if (ki) {
                    atomicOr(rem + w0, val << sh);
                    if (sh + (uint32_t)ki > 32u) atomicOr(rem + w0 + 1, val >> (32u - sh));
                }
                b += (uint32_t)ki;
            }
        }
    }
}

// Unary terminators of 8 symbols with quotients q[0..7] (ug = 8 + their sum bits in all),
// starting at bit pos of `un` (zeroed shared words).  A group whose codes fit in 32 bits is
// built in a register (last symbol first) and ORed in with at most two shared atomics.
__device__ __forceinline__ void unary_group_bits(uint32_t *un, uint32_t pos, const uint32_t (&q)[8], uint32_t ug) {
    if (ug <= 32u) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 7; i >= 0; i--) acc = ((acc << 1) | 1u) << q[i];
        const uint32_t w0 = pos >> 5, sh = pos & 31u;
        atomicOr(un + w0, acc << sh);
        if (sh) {
            const uint32_t hi = acc >> (32u - sh);
            if (hi) atomicOr(un + w0 + 1, hi);
        }
    } else {
        uint32_t p = pos;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            p += q[i];
            atomicOr(un + (p >> 5), 1u << (p & 31u));
            p += 1;
        }
    }
}
// The same, summing the group's bits; returns them.
__device__ __forceinline__ uint32_t unary_group_shared(uint32_t *un, uint32_t pos, const uint32_t (&q)[8]) {
    uint32_t ug = 8;
#pragma unroll
    for (int i = 0; i < 8; i++) ug += q[i];
    unary_group_bits(un, pos, q, ug);
    return ug;
}

// Slow path for a chunk that does not fit the stage: recompute every round and
// set each bit of the chunk (already zeroed in global memory) with an atomic;
// every access is bounded by `room` words.  Whole warp calls it.
template <int LAT, bool DITHER, bool ROT>
__device__ __noinline__ void encode_chunk_global(const EncodeArgs &a, const ChunkGeo &geo, const uint32_t *sign_tab,
                                                 const float *rot_s, uint32_t *g, unsigned long long room,
                                                 uint32_t nc, uint32_t nr) {
    const int lane = threadIdx.x & 31;
    constexpr int N = Lattice<LAT>::N;
    const int k = a.k, kl = a.k_last;
    const unsigned long long lane_bits = 4ull * group_rem_bits<N>(k, kl);   // remainder bits of 32 symbols
    const int nrounds = (geo.ntiles + kTilesPerRound - 1) / kTilesPerRound;
    unsigned long long urun = 0;
    for (int r = 0; r < nrounds; r++) {
        uint32_t z[32], cbits;
        RoundInput in;
        round_input(a, geo, r, lane, in);
        uint4 raw[4];
        {
            const uint16_t *src = nullptr;
            int tc;
            unsigned long long e;
            geo.tile(a.map, a.x, r * kTilesPerRound + (lane >> 2), src, tc, e);
#pragma unroll
            for (int j = 0; j < 4; j++)
                raw[j] = in.valid ? ldg_nc_v4(src + 32 * (lane & 3) + 8 * j) : make_uint4(0, 0, 0, 0);
        }
        uint32_t rkey;   // counted when the chunk was first encoded
        round_symbols<LAT, DITHER, ROT>(a, in, raw, lane, sign_tab, z, cbits, rkey, rot_s);
        const bool valid = in.valid;
        unsigned long long ub = 0;
#pragma unroll
        for (int i = 0; i < 32; i++) ub += z[i] >> sym_k<N>(i, k, kl);
        ub = valid ? ub + 32 : 0;
        unsigned long long incl = ub;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const unsigned long long rtot = __shfl_sync(0xffffffffu, incl, 31);
        if (valid) {
            const unsigned long long cw = 4ull * r + (lane >> 3);
            if (LAT == HQ_E8 && cbits && cw < room) atomicOr(g + cw, cbits << (4 * (lane & 7)));
            unsigned long long rb = 32ull * nc + (unsigned long long)(32 * r + lane) * lane_bits;
            unsigned long long pos = 32ull * (nc + nr) + urun + incl - ub;
            for (int i = 0; i < 32; i++) {
                const int ki = sym_k<N>(i, k, kl);
                const uint32_t rr = z[i] & ((1u << ki) - 1u);
                for (int b = 0; b < ki; b++, rb++)
                    if (((rr >> b) & 1u) && (rb >> 5) < room) atomicOr(g + (rb >> 5), 1u << (uint32_t)(rb & 31));
                pos += z[i] >> ki;
                if ((pos >> 5) < room) atomicOr(g + (pos >> 5), 1u << (uint32_t)(pos & 31));
                pos++;
            }
        }
        urun += rtot;
    }
}

// Copy a chunk's n stage words to stream[start, start + n), dropping words at or past
// cap_words: the words before the stream's first 16-byte boundary one per lane, then
// groups of four words as one 16-byte store per lane, then the last few words.  Whole
// warp.  ZERO: also clear the stage words [0, n) (forms that reuse a stage unzeroed).
template <bool ZERO>
__device__ __forceinline__ void copy_stage_out(const EncodeArgs &a, uint32_t *stream, uint32_t *stage,
                                               unsigned long long start, uint32_t n, int lane) {
    const unsigned long long cap = a.cap_words;
    uint32_t *g = stream + start;
    const uint32_t head = min(n, (uint32_t)((16u - ((uint32_t)(uintptr_t)g & 15u)) & 15u) >> 2);
    if ((uint32_t)lane < head && start + lane < cap) g[lane] = stage[lane];
    const uint32_t groups = (n - head) >> 2;
    uint4 *g4 = reinterpret_cast<uint4 *>(g + head);
    for (uint32_t q = lane; q < groups; q += 32) {
        const uint32_t s = head + 4 * q;
        const uint4 v = make_uint4(stage[s], stage[s + 1], stage[s + 2], stage[s + 3]);
        if (start + s + 4 <= cap) {
            g4[q] = v;
        } else {
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                if (start + s + j < cap) g[s + j] = w[j];
        }
    }
    const uint32_t t = head + 4 * groups + (uint32_t)lane;
    if (t < n && start + t < cap) g[t] = stage[t];
    if (ZERO) {
        __syncwarp();
        uint4 *s4 = reinterpret_cast<uint4 *>(stage);
        for (uint32_t i = lane; i < (n + 3) >> 2; i += 32) s4[i] = make_uint4(0, 0, 0, 0);
    }
}

// A chunk that has been encoded into a stage and waits for its offset.
struct Pending {
    unsigned long long c, total;
    bool overflow, range_bad;
    unsigned long long item, local;   // batch item and the chunk's index in it (0 and c unbatched)
};

// `first`: lookback_peek(a.lookback, p.c), loaded earlier so that its latency overlaps work.
// A batch item's stream is its own: its chunk offsets, tail and stream size are written
// into the item's entries, and its capacity and look-back timeout bits go straight to its
// accumulator.
template <int LAT, bool DITHER>
__device__ __forceinline__ void finish_chunk_warp(const EncodeArgs &a, const Pending &p, uint32_t *stage,
                                                  const uint32_t *sign_tab, unsigned long long base, uint32_t &status,
                                                  unsigned long long first) {
    const int lane = threadIdx.x & 31;
    const bool batched = a.batch > 1;
    const unsigned long long nloc = batched ? a.item_chunks : a.n_chunks;
    uint64_t *offs = batched ? a.offsets + p.item * (a.item_chunks + 1) : a.offsets + a.chunk_base;
    uint32_t *stream = a.stream + (batched ? p.item * a.item_stream_stride : 0ull);
    bool to = false;
    const unsigned long long excl = lookback_resolve(a.lookback, p.c, p.total, a.spin_limit, to, first, p.local == 0);
    uint32_t st = to ? HQ_ST_TIMEOUT : 0u;
    const unsigned long long start = base + excl;
    if (lane == 0) {
        offs[p.local] = start;
        if (p.local + 1 == nloc) {
            const unsigned long long end = start + p.total;
            offs[nloc] = end;
            if (a.tail_out) *a.tail_out = end;
            a.acc[p.item].stream_words = end;
            if (end > a.cap_words) st |= HQ_ST_CAPACITY;
        }
        if (p.local == 0 && a.row) *a.row = a.row_val;
        if (batched && st) atomicOr(&a.acc[p.item].status, st);
    }
    if (!batched) status |= st;
    if (!p.range_bad && !p.overflow) {
        copy_stage_out<false>(a, stream, stage, start, (uint32_t)p.total, lane);
    } else if (!p.range_bad) {
        uint32_t *g = stream + start;
        const unsigned long long room = (start < a.cap_words) ? a.cap_words - start : 0ull;
        for (unsigned long long i = lane; i < p.total; i += 32)
            if (i < room) g[i] = 0u;
        __syncwarp();
        __threadfence_block();
        ChunkGeo geo;
        geo.init(a.map, p.local);
        geo.xoff = (long long)p.item * a.item_x_stride;
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * geo.ntiles + 31) / 32u : 0u;
        const uint32_t nr = ((uint32_t)geo.ntiles * tile_rem_bits<Lattice<LAT>::N>(a.k, a.k_last) + 31u) >> 5;
        encode_chunk_global<LAT, DITHER, false>(a, geo, sign_tab, nullptr, g, room, nc, nr);
    }
    __syncwarp();
}

__device__ __forceinline__ unsigned long long take_ticket(const EncodeArgs &a) {
    unsigned long long c = 0;
    if ((threadIdx.x & 31) == 0) c = atomicAdd(a.ticket, 1u);
    return __shfl_sync(0xffffffffu, c, 0);
}

// Throughput form: persistent CTAs of kWarpsPerCta warps, each warp encoding whole
// chunks (4 rounds of 8 tiles) taken by ticket, with a two-chunk stage pipeline.
// BULK: each round's input arrives by one bulk copy (bulk_prefetch_round); otherwise
// each lane copies its own 64 bytes (prefetch_round).
// MIXED: the last symbol of each block has its own Rice parameter (a.k_last != a.k),
// so lanes' remainder runs are not word-aligned (put_rem_mixed).
// KC >= 0: the Rice parameter is KC (= a.k = a.k_last), fixed at compile time.
// KVONLY: the launch is a KV append (the weights tile map compiled out).
template <int LAT, bool DITHER, bool KSMALL, bool MIXED = false, bool BULK = false, int KC = -1, bool KVONLY = false>
__global__ void __launch_bounds__(kWarpsPerCta * 32, 2) encode_kernel(const EncodeArgs a) {
    constexpr int MAP = BULK ? kMapWeights : KVONLY ? kMapKv : kMapAny;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *sign_tab = smem;                                        // tcols * kSignWords
    uint32_t *stage_all = smem + a.tcols * kSignWords;                // warps * 2 * kStageWords
    uint32_t *in_all = stage_all + kWarpsPerCta * 2 * kStageWords;    // warps * 32 * kInSlotWords
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *stages = stage_all + warp * 2 * kStageWords;
    uint32_t *slot = in_all + (warp * 32 + lane) * kInSlotWords;
    // bulk form: the warp's 2 KB round buffer and its mbarrier (inside the warp's slots)
    uint32_t *wbuf = in_all + warp * 32 * kInSlotWords;
    const uint32_t wbuf_s = (uint32_t)__cvta_generic_to_shared(wbuf);
    const uint32_t mb = wbuf_s + kRoundBytes;
    constexpr bool bulk = BULK;
    const uint32_t *rd = bulk ? wbuf + 16 * lane : slot;
    uint32_t phase = 0;

    if (bulk && lane == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    build_sign_table(sign_tab, a.tcols, a.seed);
    __syncthreads();

    constexpr int N = Lattice<LAT>::N;
    const int k = KC >= 0 ? KC : a.k, kl = KC >= 0 ? KC : a.k_last;
    const uint32_t lane_bits = 4u * group_rem_bits<N>(k, kl);   // remainder bits of a lane's 32 symbols
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;
    uint32_t status = 0, zor_all = 0;
    unsigned long long payload = 0;
    CodeRange rng;

    unsigned long long c = take_ticket(a);
    if (c < a.n_chunks) {
        const ItemChunk ic = item_chunk<BULK>(a, c);
        ChunkGeo g0;
        g0.init<MAP, BULK>(a.map, ic.local);
        g0.xoff = (long long)ic.item * a.item_x_stride;
        if (bulk) {
            if (lane == 0) bulk_prefetch_round(a, g0, 0, wbuf_s, mb);
        } else {
            prefetch_round<MAP>(a, g0, 0, lane, slot);
        }
    }
    Pending pend;
    bool have_pend = false;
    int buf = 0;
    // a batch's stats are gathered per item: the warp's running figures belong to item
    // cur_item and are added to its accumulator when the warp moves to another item
    unsigned long long cur_item = 0;
    while (c < a.n_chunks) {
        const unsigned long long cn = take_ticket(a);
        const ItemChunk ic = item_chunk<BULK>(a, c);
        if (ic.item != cur_item) {
            stats_add_warp<LAT>(a, status, zor_all, payload, rng, cur_item);
            status = zor_all = 0;
            payload = 0;
            rng = CodeRange();
            cur_item = ic.item;
        }
        ChunkGeo geo;
        geo.init<MAP, BULK>(a.map, ic.local);
        geo.xoff = (long long)ic.item * a.item_x_stride;
        uint32_t *stage = stages + buf * kStageWords;

        const int ntiles = geo.ntiles;
        const int nrounds = (ntiles + kTilesPerRound - 1) / kTilesPerRound;
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
        const uint32_t rbits = (uint32_t)ntiles * tile_rem_bits<N>(k, kl);
        const uint32_t nr = (rbits + 31u) >> 5;
        {
            uint4 *s4 = reinterpret_cast<uint4 *>(stage);
            for (int i = lane; i < kStageWords / 4; i += 32) s4[i] = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();

        uint32_t urun = 0, zor = 0;
        bool overflow = (nc + nr) > (uint32_t)kStageWords, range_bad = false;
#pragma unroll 1
        for (int r = 0; r < nrounds; r++) {
            // this round's bytes are arriving in the lane's slot; take them, then
            // start the copy of the next round's
            RoundInput cur;
            round_input<MAP>(a, geo, r, lane, cur);
            if (bulk) {
                // a wait that gives up flags the call and waits once more (bounded) for the copy
                if (!mbar_wait(mb, phase, a.spin_limit | kBulkWaitPolls)) {
                    status |= HQ_ST_TIMEOUT;
                    mbar_wait(mb, phase, a.spin_limit | kBulkWaitPolls);
                }
                phase ^= 1u;
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            uint4 raw[4];
#pragma unroll
            for (int j = 0; j < 4; j++) raw[j] = *reinterpret_cast<const uint4 *>(rd + 4 * j);
            if (bulk) {
                __syncwarp();   // every lane has its bytes before the buffer is refilled
                if (r + 1 < nrounds) {
                    if (lane == 0) bulk_prefetch_round(a, geo, r + 1, wbuf_s, mb);
                } else if (cn < a.n_chunks) {
                    const ItemChunk icn = item_chunk<BULK>(a, cn);
                    ChunkGeo gn;
                    gn.init<MAP, BULK>(a.map, icn.local);
                    gn.xoff = (long long)icn.item * a.item_x_stride;
                    if (lane == 0) bulk_prefetch_round(a, gn, 0, wbuf_s, mb);
                }
            } else if (r + 1 < nrounds) {
                prefetch_round<MAP>(a, geo, r + 1, lane, slot);
            } else if (cn < a.n_chunks) {
                const ItemChunk icn = item_chunk<BULK>(a, cn);
                ChunkGeo gn;
                gn.init<MAP, BULK>(a.map, icn.local);
                gn.xoff = (long long)icn.item * a.item_x_stride;
                prefetch_round<MAP>(a, gn, 0, lane, slot);
            }

            uint32_t z[32], cbits, rkey;
            round_symbols<LAT, DITHER>(a, cur, raw, lane, sign_tab, z, cbits, rkey);
            rng.add<LAT>(rkey, z, cbits);
            const bool valid = cur.valid;
            // the quotients of the lane's 4 groups of 8 symbols and their sums (the unary bits)
            uint32_t qg[4][8], gsum[4], lor = 0;
#pragma unroll
            for (int g = 0; g < 4; g++) {
                gsum[g] = 8u;
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    qg[g][i] = z[8 * g + i] >> sym_k<N>(i, k, kl);
                    gsum[g] += qg[g][i];
                    lor |= z[8 * g + i];
                }
            }
            const uint32_t usum = (gsum[0] + gsum[1]) + (gsum[2] + gsum[3]) - 32u;
            zor |= lor;
            const uint32_t ub = valid ? usum + 32u : 0u;
            uint32_t incl = ub;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t rtot = __shfl_sync(0xffffffffu, incl, 31);
            const uint32_t rzor = __reduce_or_sync(0xffffffffu, lor);
            if ((rzor >> 22) != 0u || (unsigned long long)urun + rtot >= kMaxUnaryBits) range_bad = true;
            if (!overflow && nc + nr + (uint32_t)(((unsigned long long)urun + rtot + 31) >> 5) > (uint32_t)kStageWords)
                overflow = true;
            if (!overflow && !range_bad) {
                if (MIXED) {
                    if (valid) put_rem_mixed<N>(stage + nc, (uint32_t)(32 * r + lane) * lane_bits, z, k, kl);
                } else {
                    put_rem<KSMALL>(stage + nc + (uint32_t)(32 * r + lane) * (uint32_t)k, z, k, valid);
                }
                if (valid) {
                    if (LAT == HQ_E8 && cbits) atomicOr(stage + 4 * r + (lane >> 3), cbits << (4 * (lane & 7)));
                    uint32_t *un = stage + nc + nr;
                    uint32_t pos = urun + incl - ub;
#pragma unroll
                    for (int g = 0; g < 4; g++) {
                        unary_group_bits(un, pos, qg[g], gsum[g]);
                        pos += gsum[g];
                    }
                }
            }
            urun += rtot;
        }
        zor_all |= zor;
        if (range_bad) status |= HQ_ST_RANGE;
        const unsigned long long total = nc + nr + ((unsigned long long)urun + 31) / 32;
        payload += urun + (unsigned long long)rbits + ((LAT == HQ_E8) ? 16ull * ntiles : 0ull);
        lookback_publish(a.lookback, c, total, ic.local == 0);

        // the previous chunk's predecessors have had a whole chunk's time to publish
        if (have_pend)
            finish_chunk_warp<LAT, DITHER>(a, pend, stages + (buf ^ 1) * kStageWords, sign_tab, base, status,
                                           lookback_peek(a.lookback, pend.c));
        pend.c = c;
        pend.total = total;
        pend.overflow = overflow;
        pend.range_bad = range_bad;
        pend.item = ic.item;
        pend.local = ic.local;
        have_pend = true;
        c = cn;
        buf ^= 1;
    }
    if (have_pend)
        finish_chunk_warp<LAT, DITHER>(a, pend, stages + (buf ^ 1) * kStageWords, sign_tab, base, status,
                                       lookback_peek(a.lookback, pend.c));
    asm volatile("cp.async.wait_group 0;" ::: "memory");

    stats_add_warp<LAT>(a, status, zor_all, payload, rng, cur_item);
    stats_finish_cta(a);
}

// Four warps share a chunk: warp w of a group encodes round w (tiles 8w..8w+7).
constexpr int kGroupWarps = kChunkTiles / kTilesPerRound;
constexpr int kGroups = kWarpsPerCta / kGroupWarps;
static_assert(kGroups * kGroupWarps == kWarpsPerCta, "whole groups per CTA");

// Per-group control words in shared memory, double-buffered by iteration parity.
struct GroupCtl {
    uint32_t tot[2][kGroupWarps];   // unary bits of each warp's round
    uint32_t bad[2][kGroupWarps];   // nonzero: that round is outside the supported range
    unsigned int tk[2];             // ticket taken during the iteration (the chunk after next)
    unsigned int first[2];          // the group's first two tickets
};
static_assert(sizeof(GroupCtl) % 16 == 0, "keeps the input slots 16-byte aligned");

__device__ __forceinline__ void group_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(kGroupWarps * 32) : "memory");
}

// Resolve a pending chunk's offset and write it out (one warp).  The stage words
// are zeroed as they are copied, so the stage is clean for its next chunk.
template <int LAT, bool DITHER, bool ROT>
__device__ __forceinline__ void finish_chunk(const EncodeArgs &a, const Pending &p, uint32_t *stage,
                                             const uint32_t *sign_tab, const float *rot_s, unsigned long long base,
                                             uint32_t &status, unsigned long long first) {
    const int lane = threadIdx.x & 31;
    bool to = false;
    const unsigned long long excl = lookback_resolve(a.lookback, p.c, p.total, a.spin_limit, to, first, p.c == 0);
    if (to) status |= HQ_ST_TIMEOUT;
    const unsigned long long start = base + excl;
    if (lane == 0) {
        a.offsets[a.chunk_base + p.c] = start;
        if (p.c + 1 == a.n_chunks) {
            const unsigned long long end = start + p.total;
            a.offsets[a.chunk_base + a.n_chunks] = end;
            if (a.tail_out) *a.tail_out = end;
            a.acc->stream_words = end;
            if (end > a.cap_words) status |= HQ_ST_CAPACITY;
        }
        if (p.c == 0 && a.row) *a.row = a.row_val;
    }
    if (!p.range_bad && !p.overflow) {
        copy_stage_out<true>(a, a.stream, stage, start, (uint32_t)p.total, lane);
    } else if (!p.range_bad) {
        uint32_t *g = a.stream + start;
        const unsigned long long room = (start < a.cap_words) ? a.cap_words - start : 0ull;
        for (unsigned long long i = lane; i < p.total; i += 32)
            if (i < room) g[i] = 0u;
        __syncwarp();
        __threadfence_block();
        ChunkGeo geo;
        geo.init(a.map, p.c);
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * geo.ntiles + 31) / 32u : 0u;
        const uint32_t nr = ((uint32_t)geo.ntiles * tile_rem_bits<Lattice<LAT>::N>(a.k, a.k_last) + 31u) >> 5;
        encode_chunk_global<LAT, DITHER, ROT>(a, geo, sign_tab, rot_s, g, room, nc, nr);
    }
    __syncwarp();
}

// Latency form, for launches that fit in one wave of groups (a KV append, a small
// matrix): persistent CTAs of kGroups groups.  A group takes chunk tickets in increasing
// order (so a chunk's predecessors are always already running) and per chunk:
// each warp encodes its round; the four round totals meet in shared memory
// (group barrier); each warp places its codewords in the group's stage; warp 0
// publishes the chunk's word count; and one warp, in turn, resolves the previous
// chunk's offset and copies that chunk's stage out.
// ROT: the dense KV rotation instead of the sign diagonal and H_128, its shared form
// and per-warp rotation buffers (rot_smem_bytes) ahead of the rest; one CTA of
// kRotGroups groups per SM (the shared memory).  The rotation runs at the fp32 fma
// rate, so this form serves every launch size.
constexpr int kRotGroups = 3;
template <int LAT, bool DITHER, bool KSMALL, bool ROT, bool MIXED = false>
__global__ void __launch_bounds__((ROT ? kRotGroups : kGroups) * kGroupWarps * 32, ROT ? 1 : 2)
    encode_kernel_grouped(const EncodeArgs a) {
    constexpr int G = ROT ? kRotGroups : kGroups;
    extern __shared__ __align__(16) uint32_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = warp / kGroupWarps, w = warp % kGroupWarps;
    float *rot_s = ROT ? reinterpret_cast<float *>(smem) : nullptr;
    uint32_t *sign_tab = smem + (ROT ? rot_smem_bytes(G * kGroupWarps) / sizeof(uint32_t) : 0);   // tcols * kSignWords
    uint32_t *stage_all = sign_tab + a.tcols * kSignWords;                  // groups * 2 * kStageWords
    GroupCtl *ctl_all = reinterpret_cast<GroupCtl *>(stage_all + G * 2 * kStageWords);
    uint32_t *in_all = reinterpret_cast<uint32_t *>(ctl_all + G);    // warps * 32 * kGroupSlotWords
    uint32_t *stages = stage_all + gi * 2 * kStageWords;
    GroupCtl &ctl = ctl_all[gi];
    uint32_t *slot = in_all + (warp * 32 + lane) * kGroupSlotWords;

    if (ROT)
        load_rotation<true>(rot_s, a.rot);
    else
        build_sign_table(sign_tab, a.tcols, a.seed);
    for (int i = threadIdx.x; i < G * 2 * kStageWords / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(stage_all)[i] = make_uint4(0, 0, 0, 0);
    if (w == 0 && lane == 0) {
        ctl.first[0] = atomicAdd(a.ticket, 1u);
        ctl.first[1] = atomicAdd(a.ticket, 1u);
    }
    __syncthreads();

    const unsigned long long n = a.n_chunks;
    constexpr int N = Lattice<LAT>::N;
    const int k = a.k, kl = a.k_last;
    const uint32_t lane_bits = 4u * group_rem_bits<N>(k, kl);
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;
    uint32_t status = 0, zor_all = 0;
    unsigned long long payload = 0;
    CodeRange rng;
    unsigned long long c = ctl.first[0], cn = ctl.first[1];
    if (c < n) {
        ChunkGeo g0;
        g0.init(a.map, c);
        prefetch_round(a, g0, w, lane, slot);
    }
    Pending pend = {0, 0, false, false};
    bool have_pend = false;
    int buf = 0;
    unsigned it = 0;
    while (true) {
        const bool live = c < n;
        const bool duty = w == (int)(it & (kGroupWarps - 1));   // this warp finishes the previous chunk
        unsigned long long first = 0;
        if (!live && have_pend && duty) first = lookback_peek(a.lookback, pend.c);
        uint32_t *stage = stages + buf * kStageWords;
        ChunkGeo geo;
        uint32_t z[32], cbits = 0, ub = 0, incl = 0, rkey = 0;
        bool valid = false;
        if (live) {
            geo.init(a.map, c);
            RoundInput cur;
            round_input(a, geo, w, lane, cur);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            uint4 raw[4];
#pragma unroll
            for (int j = 0; j < 4; j++) raw[j] = *reinterpret_cast<const uint4 *>(slot + 4 * j);
            if (w == 0 && lane == 0) ctl.tk[buf] = atomicAdd(a.ticket, 1u);
            if (have_pend && duty) first = lookback_peek(a.lookback, pend.c);
            // the symbols are left in the lane's slot, where they wait while the group meets
            uint32_t usum, lor;
            round_symbols_rolled<LAT, DITHER, ROT>(a, cur, raw, lane, sign_tab, slot, cbits, usum, lor, rkey,
                                                   rot_s);
            valid = cur.valid;
            zor_all |= lor;
            ub = valid ? usum + 32u : 0u;
            incl = ub;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            // symbols below 2^22 keep ub below 2^28; the coarse sum says whether the
            // round's total could reach 2^31 bits (and the 32-bit scan wrap)
            const uint32_t coarse = __reduce_add_sync(0xffffffffu, ub >> 8);
            const uint32_t rzor = __reduce_or_sync(0xffffffffu, lor);
            if (lane == 31) {
                ctl.tot[buf][w] = incl;
                ctl.bad[buf][w] = ((rzor >> 22) != 0u || coarse >= (1u << 23)) ? 1u : 0u;
            }
        }
        group_sync(gi);
        unsigned long long total = 0;
        bool overflow = false, range_bad = false;
        if (live) {
            unsigned long long before = 0, U = 0;
            uint32_t badw = 0;
#pragma unroll
            for (int j = 0; j < kGroupWarps; j++) {
                const uint32_t t = ctl.tot[buf][j];
                before += (j < w) ? t : 0u;
                U += t;
                badw |= ctl.bad[buf][j];
            }
            const int ntiles = geo.ntiles;
            const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
            const uint32_t rbits = (uint32_t)ntiles * tile_rem_bits<N>(k, kl);
            const uint32_t nr = (rbits + 31u) >> 5;
            range_bad = badw != 0u || U >= kMaxUnaryBits;
            total = nc + nr + (U + 31) / 32;
            overflow = total > (unsigned long long)kStageWords;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint4 t = reinterpret_cast<const uint4 *>(slot)[j];
                z[4 * j] = t.x;
                z[4 * j + 1] = t.y;
                z[4 * j + 2] = t.z;
                z[4 * j + 3] = t.w;
            }
            rng.add<LAT>(rkey, z, cbits);
            if (cn < n) {
                ChunkGeo gn;
                gn.init(a.map, cn);
                prefetch_round(a, gn, w, lane, slot);
            }
            if (!overflow && !range_bad) {
                if (MIXED) {
                    if (valid) put_rem_mixed<N>(stage + nc, (uint32_t)(32 * w + lane) * lane_bits, z, k, kl);
                } else {
                    put_rem<KSMALL>(stage + nc + (uint32_t)(32 * w + lane) * (uint32_t)k, z, k, valid);
                }
                if (valid) {
                    if (LAT == HQ_E8 && cbits) atomicOr(stage + 4 * w + (lane >> 3), cbits << (4 * (lane & 7)));
                    uint32_t *un = stage + nc + nr;
                    uint32_t pos = (uint32_t)before + incl - ub;
#pragma unroll
                    for (int gq = 0; gq < 4; gq++) {
                        uint32_t qg[8];
#pragma unroll
                        for (int i = 0; i < 8; i++) qg[i] = z[8 * gq + i] >> sym_k<N>(i, k, kl);
                        pos += unary_group_shared(un, pos, qg);
                    }
                }
            }
            if (w == 0) {
                lookback_publish(a.lookback, c, total, c == 0);
                if (range_bad) status |= HQ_ST_RANGE;
                if (lane == 0) payload += U + (unsigned long long)rbits + ((LAT == HQ_E8) ? 16ull * ntiles : 0ull);
            }
        }
        // the previous chunk: its predecessors have had a whole chunk's time to publish
        if (have_pend && duty)
            finish_chunk<LAT, DITHER, ROT>(a, pend, stages + (buf ^ 1) * kStageWords, sign_tab, rot_s, base, status,
                                           first);
        if (!live) break;
        pend.c = c;
        pend.total = total;
        pend.overflow = overflow;
        pend.range_bad = range_bad;
        have_pend = true;
        c = cn;
        cn = ctl.tk[buf];
        buf ^= 1;
        it++;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");

    stats_add_warp<LAT>(a, status, zor_all, payload, rng);
    stats_finish_cta(a);
}


// ------------------------------------------------------------------ wide form
// Latency form for the smallest launches (a KV append of a few tokens or heads, a
// small matrix): sixteen lanes per tile, one 8-element E8 block (or 2 D4, 4 A2, 8 Z
// blocks) per lane, so a chunk's 32 tiles are spread over 16 warps, each holding
// two tiles.  A lane's serial work is a quarter of the grouped form's.
constexpr int kWideWarps = kChunkTiles / 2;   // warps per chunk, two tiles each
static_assert(kWideWarps == 16, "two tiles per warp");

struct WideCtl {
    uint32_t tot[2][kWideWarps];
    uint32_t bad[2][kWideWarps];
    unsigned int tk[2];
    unsigned int first[2];
};
static_assert(sizeof(WideCtl) % 16 == 0, "16-byte multiple");

__device__ __forceinline__ void wide_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(kWideWarps * 32) : "memory");
}

// A lane's 8 elements of its tile: signs, FWHT-128 with its 15 partner lanes (or with
// ROT the dense rotation, rot_s its shared form and xs the warp's 256-float buffer),
// scale, [+ dither], lattice blocks -> 8 zigzag symbols, (E8) the coset bit and the
// largest code key (0 for an invalid tile).
template <int LAT, bool DITHER, bool ROT = false>
__device__ __forceinline__ void wide_symbols(const EncodeArgs &a, bool valid, int tcol, unsigned long long e0,
                                             uint4 raw, int lane, const uint32_t *sign_tab, uint32_t (&z)[8],
                                             uint32_t &cbit, uint32_t &rkey, const float *rot_s = nullptr,
                                             float *xs = nullptr) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    const int l16 = lane & 15;
    const uint4 w = valid ? raw : make_uint4(0, 0, 0, 0);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    float2 v[4];
    if constexpr (ROT) {
#pragma unroll
        for (int t = 0; t < 4; t++)
            v[t] = make_float2(__uint_as_float(wv[t] << 16), __uint_as_float(wv[t] & 0xFFFF0000u));
        rotate_sixteenth(v, rot_s, xs, lane);
    } else {
        const uint32_t es = sign_tab[tcol * kSignWords + (l16 >> 2)];
#pragma unroll
        for (int t = 0; t < 4; t++) {
            const uint32_t ww = wv[t] ^ sign_pair_mask(es, 4 * (l16 & 3) + t);
            v[t] = make_float2(__uint_as_float(ww << 16), __uint_as_float(ww & 0xFFFF0000u));
        }
        fwht128_sixteenth(v, lane);
    }
    const float2 c2 = make_float2(a.c_scale, a.c_scale);
#pragma unroll
    for (int t = 0; t < 4; t++) v[t] = f2_mul(v[t], c2);
    const float x[8] = {v[0].x, v[0].y, v[1].x, v[1].y, v[2].x, v[2].y, v[3].x, v[3].y};
    cbit = 0;
    rkey = 0;
    const unsigned long long eq = e0 + 8ull * l16;
#pragma unroll
    for (int b = 0; b < 8 / N; b++) {
        float blk[N];
#pragma unroll
        for (int i = 0; i < N; i++) blk[i] = x[b * N + i];
        if (DITHER) {
            float d[N];
            dither_block<LAT>(a.seed, eq + (unsigned long long)(b * N), d);
#pragma unroll
            for (int i = 0; i < N; i++) blk[i] = __fadd_rn(blk[i], d[i]);
        }
        uint32_t zz[N];
        cbit |= L::symbols(blk, zz, rkey) << b;
#pragma unroll
        for (int i = 0; i < N; i++) z[b * N + i] = (!DITHER || valid) ? zz[i] : 0u;
    }
    if (!valid) cbit = 0;
    if (!valid) rkey = 0;
}

// k remainder bits of 8 symbols into the remainder plane at bit `off` (any
// alignment: ORed into the stage, at most two words per value group).
__device__ __forceinline__ void wide_put_rem(uint32_t *rem, uint32_t off, const uint32_t (&z)[8], int k) {
    if (k == 0) return;
    const uint32_t mask = (1u << k) - 1u;
    if (k <= 4) {
        const uint32_t pk = 1u << k;
        uint32_t gv = 0;
#pragma unroll
        for (int i = 7; i >= 0; i--) gv = imad(gv, pk, z[i] & mask);
        const uint32_t w0 = off >> 5, sh = off & 31u;
        atomicOr(rem + w0, gv << sh);
        if (sh + 8u * (uint32_t)k > 32u) atomicOr(rem + w0 + 1, gv >> (32u - sh));
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint32_t b = off + (uint32_t)(i * k), w0 = b >> 5, sh = b & 31u, val = z[i] & mask;
            atomicOr(rem + w0, val << sh);
            if (sh + (uint32_t)k > 32u) atomicOr(rem + w0 + 1, val >> (32u - sh));
        }
    }
}

// One group of 16 warps per CTA.  Per chunk: every warp encodes its two tiles; the
// 16 warp totals meet in shared memory (barrier 1); each warp places its codewords
// in the stage (the coset word of its 32 blocks by one ballot, remainder bits and
// unary terminators by shared atomics); warp 0 publishes the chunk's count; one
// warp, in turn, resolves the previous chunk's offset and copies its stage out.
template <int LAT, bool DITHER>
__global__ void __launch_bounds__(kWideWarps * 32, 1) encode_kernel_wide(const EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t *sign_tab = smem;                                         // tcols * kSignWords
    uint32_t *stages = sign_tab + a.tcols * kSignWords;                // 2 * kStageWords
    WideCtl &ctl = *reinterpret_cast<WideCtl *>(stages + 2 * kStageWords);

    build_sign_table(sign_tab, a.tcols, a.seed);
    for (int i = threadIdx.x; i < 2 * kStageWords / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(stages)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        ctl.first[0] = atomicAdd(a.ticket, 1u);
        ctl.first[1] = atomicAdd(a.ticket, 1u);
    }
    __syncthreads();

    const unsigned long long n = a.n_chunks;
    const int k = a.k;
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;
    const int ti = 2 * w + (lane >> 4);          // the lane's tile in the chunk
    uint32_t status = 0, zor_all = 0;
    unsigned long long payload = 0;
    CodeRange rng;
    unsigned long long c = ctl.first[0], cn = ctl.first[1];
    // the next chunk's 16 bytes are loaded one iteration ahead
    uint4 raw_next = make_uint4(0, 0, 0, 0);
    if (c < n) {
        ChunkGeo g0;
        g0.init(a.map, c);
        const uint16_t *src;
        int tc;
        unsigned long long e0;
        if (g0.tile(a.map, a.x, ti, src, tc, e0)) raw_next = ldg_nc_v4(src + 8 * (lane & 15));
    }
    Pending pend = {0, 0, false, false};
    bool have_pend = false;
    int buf = 0;
    unsigned it = 0;
    while (true) {
        const bool live = c < n;
        const bool duty = w == (int)(it % kWideWarps);
        unsigned long long first = 0;
        if (have_pend && duty) first = lookback_peek(a.lookback, pend.c);
        uint32_t *stage = stages + buf * kStageWords;
        ChunkGeo geo;
        uint32_t z[8], cbit = 0, ub = 0, incl = 0;
        bool valid = false;
        if (live) {
            geo.init(a.map, c);
            const uint16_t *src = nullptr;
            int tcol = 0;
            unsigned long long e0 = 0;
            valid = geo.tile(a.map, a.x, ti, src, tcol, e0);
            const uint4 raw = raw_next;
            if (cn < n) {
                ChunkGeo gn;
                gn.init(a.map, cn);
                const uint16_t *s2;
                int tc2;
                unsigned long long e2;
                raw_next = gn.tile(a.map, a.x, ti, s2, tc2, e2) ? ldg_nc_v4(s2 + 8 * (lane & 15))
                                                                : make_uint4(0, 0, 0, 0);
            }
            if (threadIdx.x == 0) ctl.tk[buf] = atomicAdd(a.ticket, 1u);
            uint32_t rkey;
            wide_symbols<LAT, DITHER>(a, valid, tcol, e0, raw, lane, sign_tab, z, cbit, rkey);
            rng.add<LAT>(rkey, z, cbit);
            uint32_t usum = 0, lor = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                usum += z[i] >> k;
                lor |= z[i];
            }
            zor_all |= lor;
            ub = valid ? usum + 8u : 0u;   // symbols below 2^22: a warp's total stays below 2^30
            incl = ub;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t rzor = __reduce_or_sync(0xffffffffu, lor);
            if (lane == 31) {
                ctl.tot[buf][w] = incl;
                ctl.bad[buf][w] = (rzor >> 22) != 0u ? 1u : 0u;
            }
        }
        wide_sync();
        unsigned long long total = 0;
        bool overflow = false, range_bad = false;
        if (live) {
            unsigned long long before = 0, U = 0;
            uint32_t badw = 0;
#pragma unroll
            for (int j = 0; j < kWideWarps; j++) {
                const uint32_t t = ctl.tot[buf][j];
                before += (j < w) ? t : 0u;
                U += t;
                badw |= ctl.bad[buf][j];
            }
            const int ntiles = geo.ntiles;
            const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
            const uint32_t nr = 4u * (uint32_t)k * (uint32_t)ntiles;
            range_bad = badw != 0u || U >= kMaxUnaryBits;
            total = nc + nr + (U + 31) / 32;
            overflow = total > (unsigned long long)kStageWords;
            if (!overflow && !range_bad) {
                if (LAT == HQ_E8) {
                    const uint32_t cw = __ballot_sync(0xffffffffu, cbit != 0u);
                    if (lane == 0 && cw) stage[w] = cw;
                }
                if (valid) {
                    wide_put_rem(stage + nc, (uint32_t)(32 * w + lane) * 8u * (uint32_t)k, z, k);
                    uint32_t qg[8];
#pragma unroll
                    for (int i = 0; i < 8; i++) qg[i] = z[i] >> k;
                    unary_group_shared(stage + nc + nr, (uint32_t)before + incl - ub, qg);
                }
            }
            if (w == 0) {
                lookback_publish(a.lookback, c, total, c == 0);
                if (range_bad) status |= HQ_ST_RANGE;
                if (lane == 0) payload += U + (unsigned long long)nr * 32 + ((LAT == HQ_E8) ? 16ull * ntiles : 0ull);
            }
        }
        if (have_pend && duty)
            finish_chunk<LAT, DITHER, false>(a, pend, stages + (buf ^ 1) * kStageWords, sign_tab, nullptr, base,
                                             status, first);
        if (!live) break;
        pend.c = c;
        pend.total = total;
        pend.overflow = overflow;
        pend.range_bad = range_bad;
        have_pend = true;
        c = cn;
        cn = ctl.tk[buf];
        buf ^= 1;
        it++;
    }

    stats_add_warp<LAT>(a, status, zor_all, payload, rng);
    stats_finish_cta(a);
}

// ------------------------------------------------------------------ single-CTA form
// For launches of a few chunks (a KV append of a few tokens: one chunk per head), the
// multi-CTA machinery costs more than the work: the ticket, the look-back across CTAs,
// the done counter and the workspace clearing before the launch.  Here one CTA of
// kTinyWarps warps does it all: warp w encodes chunks w, w + kTinyWarps, ... each into
// its own stage (the per-warp form's rounds, inputs read straight from global memory);
// one warp scans the chunk sizes into offsets; the warps copy their stages out (or
// set an oversize chunk's bits in place).  No workspace is read or written.
constexpr int kTinyWarps = 8;
constexpr int kTinyMaxChunks = 32;      // stages in shared memory: 128 KB
constexpr int kTinyMaxChunksRot = 16;   // with the dense rotation's 99 KB: 64 KB of stages

struct TinyChunk {
    uint32_t total;      // words of the chunk
    uint32_t status;     // HQ_ST_RANGE
    uint32_t overflow;   // larger than its stage: set in place after the scan
    uint32_t zor;
    unsigned long long payload;
    uint32_t key, ovf;   // the chunk's integer range of the codes (CodeRange)
};

// The single-CTA forms' last steps, after a barrier that publishes info[]: every warp
// scans the chunk sizes (at most 32) into offsets from `base` (the stream's end before
// this call, loaded at the kernel's start), so that it can copy its own stages out (or
// set an oversize chunk's bits in place) without a second barrier; warp 0 also writes
// the offsets, the tail, the append row and the stats.  Whole CTA calls it.
template <int LAT, bool DITHER, bool ROT>
__device__ __forceinline__ void tiny_finish(const EncodeArgs &a, int n, const TinyChunk *info,
                                            unsigned long long base, const uint32_t *stage_all, int stage_words,
                                            const uint32_t *sign_tab, const float *rot_s) {
    constexpr int N = Lattice<LAT>::N;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const TinyChunk mine = lane < n ? info[lane] : TinyChunk{0u, 0u, 0u, 0u, 0ull, 0u, 0u};
    unsigned long long incl = mine.total;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    const unsigned long long st_lane = base + incl - mine.total;   // chunk `lane`'s first word
    if (warp == 0) {
        if (lane < n) a.offsets[a.chunk_base + lane] = st_lane;
        const unsigned long long end = base + __shfl_sync(0xffffffffu, incl, 31);
        const uint32_t status = __reduce_or_sync(0xffffffffu, mine.status) | (end > a.cap_words ? HQ_ST_CAPACITY : 0u);
        const uint32_t zor = __reduce_or_sync(0xffffffffu, mine.zor);
        const unsigned long long payload = warp_sum_u64(mine.payload);
        const uint32_t am = code_abs_of_key<LAT>(__reduce_max_sync(0xffffffffu, mine.key));
        const unsigned long long ovf = warp_sum_u64(mine.ovf);
        if (lane == 0) {
            a.offsets[a.chunk_base + n] = end;
            if (a.tail_out) *a.tail_out = end;
            if (a.row) *a.row = a.row_val;
            if (a.stats) {
                if (a.stats_add) {
                    if (status) atomicOr(&a.stats->status, status);
                    if (zor) atomicOr(&a.stats->max_symbol, zor);
                    if (payload) atomicAdd((unsigned long long *)&a.stats->payload_bits, payload);
                    if (am) atomicMax(&a.stats->max_abs_code, am);
                    if (ovf) atomicAdd((unsigned long long *)&a.stats->int8_overflow_count, ovf);
                } else {
                    a.stats->status = status;
                    a.stats->max_symbol = zor;
                    a.stats->payload_bits = payload;
                    a.stats->max_abs_code = am;
                    a.stats->reserved = 0u;
                    a.stats->int8_overflow_count = ovf;
                }
                a.stats->stream_words = end;
            }
        }
    }

    for (int c = warp; c < n; c += kTinyWarps) {   // warp-uniform
        const TinyChunk t = info[c];
        const unsigned long long st = __shfl_sync(0xffffffffu, st_lane, c);
        if (t.status) continue;   // outside the supported range: nothing written
        if (!t.overflow) {
            const uint32_t *stage = stage_all + c * stage_words;
            for (uint32_t i = lane; i < t.total; i += 32)
                if (st + i < a.cap_words) a.stream[st + i] = stage[i];
        } else {
            uint32_t *g = a.stream + st;
            const unsigned long long room = (st < a.cap_words) ? a.cap_words - st : 0ull;
            for (unsigned long long i = lane; i < t.total; i += 32)
                if (i < room) g[i] = 0u;
            __syncwarp();
            __threadfence_block();
            ChunkGeo geo;
            geo.init(a.map, (unsigned long long)c);
            const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * geo.ntiles + 31) / 32u : 0u;
            const uint32_t nr = ((uint32_t)geo.ntiles * tile_rem_bits<N>(a.k, a.k_last) + 31u) >> 5;
            encode_chunk_global<LAT, DITHER, ROT>(a, geo, sign_tab, rot_s, g, room, nc, nr);
        }
    }
}

template <int LAT, bool DITHER, bool KSMALL, bool ROT, bool MIXED>
__global__ void __launch_bounds__(kTinyWarps * 32, 1) encode_kernel_tiny(const EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int N = Lattice<LAT>::N;
    constexpr int kMax = ROT ? kTinyMaxChunksRot : kTinyMaxChunks;
    float *rot_s = ROT ? reinterpret_cast<float *>(smem) : nullptr;
    uint32_t *sign_tab = smem + (ROT ? kRotSmemBytes / sizeof(uint32_t) : 0);   // tcols * kSignWords
    uint32_t *stage_all = sign_tab + a.tcols * kSignWords;                         // kMax * kStageWords
    TinyChunk *info = reinterpret_cast<TinyChunk *>(stage_all + kMax * kStageWords);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = (int)a.n_chunks;   // <= kMax (host)
    // the stream's end before this call (the previous append's tail), loaded now so that its
    // latency passes under the encoding
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;

    if (ROT)
        load_rotation<true>(rot_s, a.rot);
    else
        build_sign_table(sign_tab, a.tcols, a.seed);
    for (int i = threadIdx.x; i < n * kStageWords / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(stage_all)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    const int k = a.k, kl = a.k_last;
    const uint32_t lane_bits = 4u * group_rem_bits<N>(k, kl);
    for (int c = warp; c < n; c += kTinyWarps) {
        ChunkGeo geo;
        geo.init(a.map, (unsigned long long)c);
        uint32_t *stage = stage_all + c * kStageWords;
        const int ntiles = geo.ntiles;
        const int nrounds = (ntiles + kTilesPerRound - 1) / kTilesPerRound;
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
        const uint32_t rbits = (uint32_t)ntiles * tile_rem_bits<N>(k, kl);
        const uint32_t nr = (rbits + 31u) >> 5;
        uint32_t urun = 0, zor = 0;
        CodeRange rng;
        bool overflow = (nc + nr) > (uint32_t)kStageWords, range_bad = false;
#pragma unroll 1
        for (int r = 0; r < nrounds; r++) {
            RoundInput in;
            round_input(a, geo, r, lane, in);
            uint4 raw[4];
            {
                const uint16_t *src = nullptr;
                int tc;
                unsigned long long e;
                geo.tile(a.map, a.x, r * kTilesPerRound + (lane >> 2), src, tc, e);
#pragma unroll
                for (int j = 0; j < 4; j++)
                    raw[j] = in.valid ? ldg_nc_v4(src + 32 * (lane & 3) + 8 * j) : make_uint4(0, 0, 0, 0);
            }
            uint32_t z[32], cbits, rkey;
            round_symbols<LAT, DITHER, ROT>(a, in, raw, lane, sign_tab, z, cbits, rkey, rot_s);
            rng.add<LAT>(rkey, z, cbits);
            const bool valid = in.valid;
            uint32_t usum = 0, lor = 0;
#pragma unroll
            for (int i = 0; i < 32; i++) {
                usum += z[i] >> sym_k<N>(i, k, kl);
                lor |= z[i];
            }
            zor |= lor;
            const uint32_t ub = valid ? usum + 32u : 0u;
            uint32_t incl = ub;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t rtot = __shfl_sync(0xffffffffu, incl, 31);
            const uint32_t rzor = __reduce_or_sync(0xffffffffu, lor);
            if ((rzor >> 22) != 0u || (unsigned long long)urun + rtot >= kMaxUnaryBits) range_bad = true;
            if (!overflow && nc + nr + (uint32_t)(((unsigned long long)urun + rtot + 31) >> 5) > (uint32_t)kStageWords)
                overflow = true;
            if (!overflow && !range_bad) {
                if (MIXED) {
                    if (valid) put_rem_mixed<N>(stage + nc, (uint32_t)(32 * r + lane) * lane_bits, z, k, kl);
                } else {
                    put_rem<KSMALL>(stage + nc + (uint32_t)(32 * r + lane) * (uint32_t)k, z, k, valid);
                }
                if (valid) {
                    if (LAT == HQ_E8 && cbits) atomicOr(stage + 4 * r + (lane >> 3), cbits << (4 * (lane & 7)));
                    uint32_t *un = stage + nc + nr;
                    uint32_t pos = urun + incl - ub;
#pragma unroll
                    for (int g = 0; g < 4; g++) {
                        uint32_t qg[8];
#pragma unroll
                        for (int i = 0; i < 8; i++) qg[i] = z[8 * g + i] >> sym_k<N>(i, k, kl);
                        pos += unary_group_shared(un, pos, qg);
                    }
                }
            }
            urun += rtot;
        }
        zor = __reduce_or_sync(0xffffffffu, zor);
        const uint32_t ckey = __reduce_max_sync(0xffffffffu, rng.key);
        const uint32_t covf = __reduce_add_sync(0xffffffffu, rng.ovf);
        if (lane == 0) {
            TinyChunk t;
            t.key = ckey;
            t.ovf = covf;
            t.total = nc + nr + (uint32_t)(((unsigned long long)urun + 31) / 32);
            t.status = range_bad ? HQ_ST_RANGE : 0u;
            t.overflow = overflow ? 1u : 0u;
            t.zor = zor;
            t.payload = urun + (unsigned long long)rbits + ((LAT == HQ_E8) ? 16ull * ntiles : 0ull);
            info[c] = t;
        }
        __syncwarp();
    }
    __syncthreads();

    tiny_finish<LAT, DITHER, ROT>(a, n, info, base, stage_all, kStageWords, sign_tab, rot_s);
}

// One-token KV appends (every chunk one tile: one token of one head), up to kTinyMaxChunks
// chunks: the single-CTA form, with each half-warp encoding one chunk in the wide form's
// layout (16 lanes to the tile, one 8-element lattice block each).  A lane then carries
// one lattice block and one dither block instead of four, which shortens the chain that
// sets a decode step's append latency.  The chunk's unary bits are placed by a scan over
// its 16 lanes; its stage is kTokStageWords long (larger chunks take the in-place path).
// With ROT the dense rotation replaces the sign diagonal and H_128 (each lane computes
// its 8 outputs in full, rotate_sixteenth).  Single Rice parameter only.
constexpr int kTokStageWords = 256;

template <int LAT, bool DITHER, bool ROT>
__global__ void __launch_bounds__(kTinyWarps * 32, 1) encode_kernel_tok(const EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    float *rot_s = ROT ? reinterpret_cast<float *>(smem) : nullptr;   // rot_smem_bytes(kTinyWarps)
    uint32_t *sign_tab = smem + (ROT ? rot_smem_bytes(kTinyWarps) / sizeof(uint32_t) : 0);   // tcols * kSignWords
    uint32_t *stage_all = sign_tab + a.tcols * kSignWords;           // kTinyMaxChunks * kTokStageWords
    TinyChunk *info = reinterpret_cast<TinyChunk *>(stage_all + kTinyMaxChunks * kTokStageWords);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, l16 = lane & 15;
    const int n = (int)a.n_chunks;   // <= kTinyMaxChunks, one tile each (host)
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;   // early, as in the single-CTA form

    if (ROT)
        load_rotation<true>(rot_s, a.rot);
    else
        build_sign_table(sign_tab, a.tcols, a.seed);
    // with ROT: the first 256 floats of the warp's rotation buffer hold its two tiles
    float *xs = ROT ? rot_s + 128 * kRotPitch + warp * kRotBufFloats : nullptr;
    for (int i = threadIdx.x; i < n * kTokStageWords / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(stage_all)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    const int k = a.k;
    const uint32_t nc = (LAT == HQ_E8) ? 1u : 0u;   // the coset word of the tile's 16 blocks
    const uint32_t nr = 4u * (uint32_t)k;           // 128 remainders of k bits
    for (int c0 = 2 * warp; c0 < n; c0 += 2 * kTinyWarps) {
        const int c = c0 + (lane >> 4);
        const bool live = c < n;
        const uint16_t *src = nullptr;
        int tcol = 0;
        unsigned long long e0 = 0;
        bool valid = false;
        if (live) {
            ChunkGeo geo;
            geo.init(a.map, (unsigned long long)c);
            valid = geo.tile(a.map, a.x, 0, src, tcol, e0);
        }
        const uint4 raw = valid ? ldg_nc_v4(src + 8 * l16) : make_uint4(0, 0, 0, 0);
        uint32_t z[8], cbit, rkey;
        wide_symbols<LAT, DITHER, ROT>(a, valid, tcol, e0, raw, lane, sign_tab, z, cbit, rkey, rot_s, xs);
        CodeRange rng;
        rng.add<LAT>(rkey, z, cbit);
        uint32_t usum = 0, hz = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            usum += z[i] >> k;
            hz |= z[i];
        }
        const uint32_t ub = valid ? usum + 8u : 0u;
        uint32_t incl = ub;   // within the half-warp
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (l16 >= o) incl += t;
        }
        const uint32_t U = __shfl_sync(0xffffffffu, incl, lane | 15);
#pragma unroll
        for (int o = 8; o; o >>= 1) {
            hz |= __shfl_xor_sync(0xffffffffu, hz, o);
            rng.key = max(rng.key, __shfl_xor_sync(0xffffffffu, rng.key, o));
            rng.ovf += __shfl_xor_sync(0xffffffffu, rng.ovf, o);
        }
        const bool range_bad = (hz >> 22) != 0u || U >= kMaxUnaryBits;
        const uint32_t total = nc + nr + (U + 31u) / 32u;
        const bool overflow = total > (uint32_t)kTokStageWords;
        const uint32_t cw = __ballot_sync(0xffffffffu, cbit != 0u);
        if (valid && !overflow && !range_bad) {
            uint32_t *stage = stage_all + c * kTokStageWords;
            if (LAT == HQ_E8 && l16 == 0) {
                const uint32_t bits = (lane & 16) ? (cw >> 16) : (cw & 0xFFFFu);
                if (bits) stage[0] = bits;
            }
            wide_put_rem(stage + nc, (uint32_t)l16 * 8u * (uint32_t)k, z, k);
            uint32_t qg[8];
#pragma unroll
            for (int i = 0; i < 8; i++) qg[i] = z[i] >> k;
            unary_group_shared(stage + nc + nr, incl - ub, qg);
        }
        if (live && l16 == 0) {
            TinyChunk t;
            t.total = total;
            t.status = range_bad ? HQ_ST_RANGE : 0u;
            t.overflow = overflow ? 1u : 0u;
            t.zor = hz;
            t.payload = U + 128ull * (unsigned long long)k + ((LAT == HQ_E8) ? 16ull : 0ull);
            t.key = rng.key;
            t.ovf = rng.ovf;
            info[c] = t;
        }
    }
    __syncthreads();

    tiny_finish<LAT, DITHER, ROT>(a, n, info, base, stage_all, kTokStageWords, sign_tab, rot_s);
}

// ------------------------------------------------------------------ rate only
// The quantize path up to the Rice code lengths, without a stream: per chunk the
// unary bits U, so payload = U + remainder bits + coset bits and the chunk's words
// = coset + remainder + ceil(U / 32), exactly as the encoder counts them.  Chunks
// are independent here (no offsets), so warps take them by a static stride.
template <int LAT, bool DITHER, bool ROT>
__global__ void __launch_bounds__(kWarpsPerCta * 32, ROT ? 1 : 2) rate_kernel(const EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    float *rot_s = ROT ? reinterpret_cast<float *>(smem) : nullptr;
    uint32_t *sign_tab = smem + (ROT ? kRotSmemBytes / sizeof(uint32_t) : 0);
    if (ROT)
        load_rotation<true>(rot_s, a.rot);
    else
        build_sign_table(sign_tab, a.tcols, a.seed);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    constexpr int N = Lattice<LAT>::N;
    const int k = a.k, kl = a.k_last;
    const unsigned long long nwarps = (unsigned long long)gridDim.x * kWarpsPerCta;
    unsigned long long payload = 0, words = 0;
    uint32_t status = 0, zor_all = 0;
    CodeRange rng;
    for (unsigned long long c = (unsigned long long)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); c < a.n_chunks;
         c += nwarps) {
        ChunkGeo geo;
        geo.init(a.map, c);
        const int nrounds = (geo.ntiles + kTilesPerRound - 1) / kTilesPerRound;
        unsigned long long U = 0;
        uint32_t lor = 0;
#pragma unroll 1
        for (int r = 0; r < nrounds; r++) {
            RoundInput in;
            const uint16_t *src = nullptr;
            in.tcol = 0;
            in.e0 = 0;
            in.valid = geo.tile(a.map, a.x, r * kTilesPerRound + (lane >> 2), src, in.tcol, in.e0);
            uint4 raw[4];
#pragma unroll
            for (int j = 0; j < 4; j++)
                raw[j] = in.valid ? ldg_nc_v4(src + 32 * (lane & 3) + 8 * j) : make_uint4(0, 0, 0, 0);
            uint32_t z[32], cbits, rkey;
            round_symbols<LAT, DITHER, ROT>(a, in, raw, lane, sign_tab, z, cbits, rkey, rot_s);
            rng.add<LAT>(rkey, z, cbits);
            uint32_t usum = 0;
#pragma unroll
            for (int i = 0; i < 32; i++) {
                usum += z[i] >> sym_k<N>(i, k, kl);
                lor |= z[i];
            }
            // symbols below 2^22 keep ub below 2^28: two 32-bit sums of its halves are exact
            const uint32_t ub = in.valid ? usum + 32u : 0u;
            const uint32_t lo = __reduce_add_sync(0xffffffffu, ub & 0xFFFFu);
            const uint32_t hi = __reduce_add_sync(0xffffffffu, ub >> 16);
            U += (unsigned long long)lo + ((unsigned long long)hi << 16);
        }
        lor = __reduce_or_sync(0xffffffffu, lor);
        zor_all |= lor;
        const unsigned long long nc = (LAT == HQ_E8) ? (16ull * geo.ntiles + 31) / 32 : 0ull;
        const unsigned long long rbits = (unsigned long long)geo.ntiles * tile_rem_bits<N>(k, kl);
        const unsigned long long nr = (rbits + 31) / 32;
        payload += U + rbits + ((LAT == HQ_E8) ? 16ull * geo.ntiles : 0ull);
        words += nc + nr + (U + 31) / 32;
        if ((lor >> 22) != 0u || U >= kMaxUnaryBits) status |= HQ_ST_RANGE;
    }
    const uint32_t key = __reduce_max_sync(0xffffffffu, rng.key);
    const uint32_t ovf = __reduce_add_sync(0xffffffffu, rng.ovf);
    if (lane == 0) {
        if (status) atomicOr(&a.stats->status, status);
        if (zor_all) atomicOr(&a.stats->max_symbol, zor_all);
        if (payload) atomicAdd((unsigned long long *)&a.stats->payload_bits, payload);
        if (words) atomicAdd((unsigned long long *)&a.stats->stream_words, words);
        if (key) atomicMax(&a.stats->max_abs_code, code_abs_of_key<LAT>(key));
        if (ovf) atomicAdd((unsigned long long *)&a.stats->int8_overflow_count, (unsigned long long)ovf);
    }
}


}  // namespace
}  // namespace hq
