// hq_decode.cuh -- the decode + dequantize kernel (HyperQuant "Methodology"
// sections 1-4 inverted): Rice planes -> symbols -> re-inserted membership bits
// -> lattice point [- dither] -> scale -> FWHT-128 -> sign, and then one of three
// outputs: the bf16 or fp32 tile (hq_dequantize, hq_kv_read), the tile's dot
// product with a bf16 vector (hq_gemv: one partial per tile), or a KV tile's dot
// products with the query heads of its group (hq_kv_scores).  Included by
// hq_decode.cu (stored tiles) and hq_consume.cu (dot products), each of which
// instantiates the modes it launches.
//
// Work decomposition (B200, sm_100a):
//  * a chunk (32 tiles) decodes in 4 rounds of 8 tiles, four lanes to a tile and
//    32 symbols / elements to a lane; a warp decodes whole chunks, strided over
//    the grid, unless the launch has at most half as many chunks as the grid has
//    warps: then two or four warps share a chunk, two rounds or one each, so a
//    short launch still reaches every SM;
//  * the chunk's words are brought into a per-warp shared-memory stage with
//    cp.async while the warp is still decoding the previous chunk (two stages
//    per warp); chunks too large for a stage are read from global memory;
//  * the lanes split the unary plane into 32 word ranges, count terminators
//    (popc) and scan, so every 32-symbol segment learns where its first
//    codeword starts; each lane then reads its 32 quotients from bit-reversed
//    32-bit windows, four symbols per window (one count-leading-zeros and one
//    shift per symbol), its k remainder bits from its own fixed region, and
//    rebuilds and scales the lattice points;
//  * the inverse FWHT runs in registers (two stages across the four lanes by
//    shuffle), followed by the sign flip and 16-byte stores; or, for a KV cache
//    with the dense rotation, x = Q^T z with Q^T in shared memory (rotate_round).
// Chunks are independent (their offsets are given), so there is no look-back; a
// chunk shared by several warps is staged and scanned by each.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_device.cuh"

namespace hq {

namespace {

constexpr int kStagePad = 4;   // zero words after a staged chunk: unchecked 2-word reads stay inside
constexpr int kRotDecodeWarps = 12;   // warps per CTA of the dense-rotation decoder (one CTA per SM)
constexpr int kRoundsPerChunk = 32 / kTilesPerRound;   // the decoder's unit of work is one round

// 32 bits of a plane of `n` words starting at bit `b`; words at or past n read as 0.
__device__ __forceinline__ uint32_t fetch32_checked(const uint32_t *p, uint32_t n, uint32_t b) {
    const uint32_t w = b >> 5;
    const uint32_t a0 = (w < n) ? p[w] : 0u;
    const uint32_t a1 = (w + 1 < n) ? p[w + 1] : 0u;
    return __funnelshift_r(a0, a1, b & 31u);
}

// The same from a staged chunk: the stage is zero-padded after the chunk and
// the word index is clamped to the plane's end, so both reads stay inside.
__device__ __forceinline__ uint32_t fetch32_staged(const uint32_t *p, uint32_t n, uint32_t b) {
    const uint32_t w = min(b >> 5, n);
    return __funnelshift_r(p[w], p[w + 1], b & 31u);
}

template <bool STAGED>
__device__ __forceinline__ uint32_t fetch32(const uint32_t *p, uint32_t n, uint32_t b) {
    return STAGED ? fetch32_staged(p, n, b) : fetch32_checked(p, n, b);
}

// Bit index of the n-th (0-based) set bit of w (n < popc(w)): binary search on
// popcounts of the low halves, branch-free.
__device__ __forceinline__ uint32_t select_bit(uint32_t w, uint32_t n) {
    uint32_t pos = 0, c;
    c = __popc(w & 0xFFFFu); if (n >= c) { n -= c; pos += 16; w >>= 16; }
    c = __popc(w & 0xFFu);   if (n >= c) { n -= c; pos += 8;  w >>= 8; }
    c = __popc(w & 0xFu);    if (n >= c) { n -= c; pos += 4;  w >>= 4; }
    c = __popc(w & 0x3u);    if (n >= c) { n -= c; pos += 2;  w >>= 2; }
    c = w & 1u;              if (n >= c) { pos += 1; }
    return pos;
}

// Slow path of the unary reader: 4 quotients read one terminator at a time
// (quotients may exceed the 32-bit window).  Out of line: rare.  Returns the
// new bit position; *ok turns false if the plane ends early.
__device__ __noinline__ uint32_t unary_slow(const uint32_t *un, uint32_t nu, uint32_t bp, bool *ok, uint32_t *q) {
    const uint32_t nbits = nu * 32u;
    for (int i = 0; i < 4; i++) {
        uint32_t t = 0;
        uint32_t x = __brev(fetch32_checked(un, nu, bp));
        while (x == 0u && *ok) {
            t += 32u;
            bp += 32u;
            if (bp >= nbits) *ok = false;
            x = __brev(fetch32_checked(un, nu, bp));
        }
        const uint32_t c = __clz(x);
        q[i] = t + c;
        bp += c + 1u;
    }
    return bp;
}

// Quotients of 4 symbols from bit bp of the unary plane: the next 32 stream
// bits bit-reversed (first bit at the MSB); if they hold 4 terminators each
// quotient is a count-leading-zeros, else the slow path.
template <bool STAGED>
__device__ __forceinline__ void unary4(const uint32_t *un, uint32_t nu, uint32_t &bp, bool &ok, uint32_t *q) {
    const uint32_t w = __brev(fetch32<STAGED>(un, nu, bp));
    // quotient i is the count of leading zeros after the first s_i bits, s_i = the bits of
    // the codewords before it (each quotient plus its terminator).  The shift saturates at 32
    // (w << 32 = 0, clz 32), so a window with fewer than 4 terminators ends with s > 32:
    // the check comes after the counts, with no population count first.
    uint32_t s = 0, t[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        t[i] = __clz(__funnelshift_lc(0u, w, s));
        s += t[i] + 1u;
    }
    if (s <= 32u) {
#pragma unroll
        for (int i = 0; i < 4; i++) q[i] = t[i];
        bp += s;
    } else {
        uint32_t tmp[4];
        bp = unary_slow(un, nu, bp, &ok, tmp);
#pragma unroll
        for (int i = 0; i < 4; i++) q[i] = tmp[i];
    }
}

// k-bit remainders of group g (8 symbols) from the lane's region `rw` (k words per
// 32 symbols), for k > 4: one bounded read per symbol.
__device__ __forceinline__ void rem_group(const uint32_t *rw, int k, int g, uint32_t (&r)[8]) {
    const uint32_t n = (uint32_t)k;
    const uint32_t mask = (1u << k) - 1u;
    const uint32_t b = (uint32_t)(8 * g) * (uint32_t)k;
#pragma unroll
    for (int i = 0; i < 8; i++) r[i] = fetch32_checked(rw, n, b + (uint32_t)(i * k)) & mask;
}

// The four 32-bit remainder windows of a lane (k <= 4: group g's 8k bits start at
// bit 8gk of the lane's k words), read once: k loads instead of eight, and no
// bank conflicts between lanes whose regions are k words apart.
__device__ __forceinline__ void rem_windows(const uint32_t *rw, int k, uint32_t (&x)[4]) {
    switch (k) {
    case 1: {
        const uint32_t w0 = rw[0];
        x[0] = w0; x[1] = w0 >> 8; x[2] = w0 >> 16; x[3] = w0 >> 24;
        break;
    }
    case 2: {
        const uint32_t w0 = rw[0], w1 = rw[1];
        x[0] = w0; x[1] = __funnelshift_r(w0, w1, 16); x[2] = w1; x[3] = w1 >> 16;
        break;
    }
    case 3: {
        const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
        x[0] = w0; x[1] = __funnelshift_r(w0, w1, 24); x[2] = __funnelshift_r(w1, w2, 16); x[3] = w2 >> 8;
        break;
    }
    default: {
        x[0] = rw[0]; x[1] = rw[1]; x[2] = rw[2]; x[3] = rw[3];
        break;
    }
    }
}

// Remainders of group g (8 symbols) of a lane whose 32 remainders start at bit `lb`
// of the remainder plane `rem` (nr words), with the last symbol of each lattice block
// taking kl bits and the others k (sym_k).  A group of at most 32 bits is one window.
template <int N, bool STAGED>
__device__ __forceinline__ void rem_group_mixed(const uint32_t *rem, uint32_t nr, uint32_t lb, int g, int k, int kl,
                                                uint32_t gbits, uint32_t (&r)[8]) {
    uint32_t b = lb + (uint32_t)g * gbits;
    if (gbits <= 32u) {
        uint32_t x = gbits ? fetch32<STAGED>(rem, nr, b) : 0u;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int ki = sym_k<N>(i, k, kl);
            r[i] = x & ((1u << ki) - 1u);
            x >>= ki;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int ki = sym_k<N>(i, k, kl);
            r[i] = fetch32<STAGED>(rem, nr, b) & ((1u << ki) - 1u);
            b += (uint32_t)ki;
        }
    }
}

// Where the tiles of one chunk go (computed once per chunk).
template <bool KV>
struct ChunkOut {
    int ntiles;
    float e_scale;
    long long row0, h, tok_base, tok0;
    int tc0, tpr;
    long long out_off;   // elements from out to this chunk's matrix (a batch item; 0 otherwise)

    // c: the chunk's index within its matrix; item: its batch item (weights only)
    __device__ __forceinline__ void init(const DecodeArgs &a, unsigned long long c, unsigned long long item = 0) {
        out_off = (long long)item * a.item_out_stride;
        if (KV) {
            // the append that holds global chunk c (binary search on first_chunk)
            unsigned long long lo = 0, hi = a.n_appends - 1;
            while (lo < hi) {
                const unsigned long long mid = (lo + hi + 1) >> 1;
                if (a.table[mid].first_chunk <= c) lo = mid; else hi = mid - 1;
            }
            const hq_kv_append_row row = a.table[lo];
            const long long T = row.tokens, cph = (T + 31) / 32;
            unsigned long long hq_, rq;
            divmod_u64(c - row.first_chunk, (unsigned long long)cph, hq_, rq);
            h = (long long)hq_;
            tok_base = (long long)rq * 32;
            tok0 = row.token0;
            const long long left = T - tok_base;
            ntiles = (int)(left < 32 ? left : 32);
            e_scale = row.scale_inv;
        } else {
            // a weights launch has at most 2^27 chunks (the API's limit): 32 c fits 32 bits
            tpr = (int)(a.map.cols / kTile);
            const long long t0 = (long long)c * 32, all = a.map.rows * (long long)tpr;
            ntiles = (int)((all - t0) < 32 ? (all - t0) : 32);
            const uint32_t rq = (uint32_t)t0 / (uint32_t)tpr;
            row0 = rq;
            tc0 = (int)((uint32_t)t0 - rq * (uint32_t)tpr);
            e_scale = a.e_scale;
        }
    }
    // Tile ti of the chunk: destination of its element 0 (null if not stored), sign
    // column, dither counter of element 0, and its position for dot-product outputs
    // (weights: row * tiles per row + tile column; KV: the token, or -1 past len).
    template <int MODE = kStoreTiles>
    __device__ __forceinline__ bool tile(const DecodeArgs &a, int ti, char *&dst, int &tcol,
                                         unsigned long long &e0, long long &pos) const {
        dst = nullptr;
        pos = -1;
        if (ti >= ntiles) return false;
        const size_t esz = (MODE != kStoreBf16 && a.out_fp32) ? 4 : 2;
        if (KV) {
            const long long gt = tok0 + tok_base + ti;
            tcol = 0;
            e0 = (unsigned long long)((gt * a.map.heads + h) * kTile);
            if (gt < a.len) {
                pos = gt;
                if (a.out) dst = (char *)a.out + (size_t)(h * a.out_ld_head + gt * a.out_ld) * esz;
            }
            return true;
        }
        int tc = tc0 + ti;
        long long r = row0;
        if (tc >= tpr) {
            const int d = tc / tpr;
            r += d;
            tc -= d * tpr;
        }
        tcol = tc;
        e0 = (unsigned long long)(r * a.map.cols + (long long)tc * kTile);
        pos = r * tpr + tc;
        if (a.out) dst = (char *)a.out + (size_t)(out_off + r * a.out_ld + (long long)tc * kTile) * esz;
        return true;
    }
};

// Valid word range of chunk c, or nw = 0 if the offsets are not consistent; src is the
// chunk's first word.  In a strided batch, c is split into its item and its index there.
struct ChunkWords {
    unsigned long long w0, nw;
    bool ok;
    const uint32_t *src;
    unsigned long long item, local;
};

__device__ __forceinline__ ChunkWords chunk_words(const DecodeArgs &a, unsigned long long c) {
    ChunkWords r;
    r.item = 0;
    r.local = c;
    if (a.batch > 1) {
        // a strided batch has at most 2^27 chunks in all (the API's limit)
        const uint32_t q = (uint32_t)c / (uint32_t)a.item_chunks;
        r.item = q;
        r.local = (uint32_t)c - q * (uint32_t)a.item_chunks;
    }
    const uint64_t *offs = a.offsets + r.item * (a.batch > 1 ? a.item_chunks + 1 : 0ull);
    r.w0 = offs[r.local];
    const unsigned long long w1 = offs[r.local + 1];
    r.ok = r.w0 <= w1 && w1 <= a.stream_words;
    r.nw = r.ok ? w1 - r.w0 : 0ull;
    r.src = a.stream + r.item * a.item_stream_stride + r.w0;
    return r;
}

// Start the copy of a chunk's words into a stage (cp.async, 4 bytes per lane and
// step) and zero the pad after them; one commit group per call.
__device__ __forceinline__ void stage_chunk(const DecodeArgs &a, const ChunkWords &cw, uint32_t *stage, int lane) {
    if (cw.nw <= (unsigned long long)kStageWords) {
        const uint32_t n = (uint32_t)cw.nw;
        const uint32_t *src = cw.src;
        for (uint32_t i = lane; i < n; i += 32) {
            const unsigned sa = (unsigned)__cvta_generic_to_shared(stage + i);
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(src + i) : "memory");
        }
        if (lane < kStagePad) stage[n + lane] = 0u;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// First unary bit of every 32-symbol segment of a chunk (startbit[s]): the
// lanes split the unary plane into 32 word ranges, count terminators (popc),
// scan, and each lane locates the segment boundaries that fall in its range.
// Returns false (chunk corrupt) unless the plane holds exactly nsym terminators.
__device__ __forceinline__ bool find_segment_starts(const uint32_t *un, uint32_t nu, uint32_t nsym, uint32_t nseg,
                                                    bool ok, uint32_t *startbit, int lane) {
    const uint32_t seg = (nu + 31u) / 32u;
    const uint32_t s0 = min(nu, (uint32_t)lane * seg), s1 = min(nu, s0 + seg);
    uint32_t cnt = 0;
    for (uint32_t i = s0; i < s1; i++) cnt += __popc(un[i]);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t ones = __shfl_sync(0xffffffffu, incl, 31);
    ok = ok && ones == nsym;
    if (ok) {
        const uint32_t before = incl - cnt;
        // terminator j = 32 s - 1 closes segment s - 1; find those inside [before, incl)
        uint32_t ss = (before + 1u + 31u) / 32u;
        if (ss == 0) ss = 1;
        uint32_t i = s0, seen = before;
        for (; ss < nseg && 32u * ss - 1u < incl; ss++) {
            const uint32_t j = 32u * ss - 1u;
            uint32_t w = un[i], pc = __popc(w);
            while (seen + pc <= j) {
                seen += pc;
                i++;
                w = un[i];
                pc = __popc(w);
            }
            startbit[ss] = i * 32u + select_bit(w, j - seen) + 1u;
        }
        if (lane == 0) startbit[0] = 0;
    }
    __syncwarp();
    return ok;
}

// Dot product of a lane's 32 decoded values (bf16-rounded, signs applied: exactly the
// stored bf16 tile) with 32 bf16 values of v: sequential fma in element order (the
// products of two bf16 values are exact in fp32).
__device__ __forceinline__ float lane_dot(const uint32_t (&w)[16], const uint16_t *v) {
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint4 x = ldg_nc_v4(v + 8 * j);
        const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int t = 0; t < 4; t++) {
            const uint32_t ww = w[4 * j + t];
            acc = __fmaf_rn(__uint_as_float(ww << 16), __uint_as_float(xv[t] << 16), acc);
            acc = __fmaf_rn(__uint_as_float(ww & 0xFFFF0000u), __uint_as_float(xv[t] & 0xFFFF0000u), acc);
        }
    }
    return acc;
}

// Sum over the four lanes of a tile, the same in all four: (a0 + a1) + (a2 + a3).
__device__ __forceinline__ float tile_sum(float acc) {
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    return __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
}

// Rounds [r0, r1) of one chunk, reading its planes from `src` (a stage when STAGED).
// ROT: the dense KV rotation's inverse (rot_s: its shared form) in place of H_128
// and the sign diagonal.
template <int LAT, bool DITHER, bool KV, bool KSMALL, bool STAGED, int MODE, bool ROT, bool MIXED, int KC = -1>
__device__ __forceinline__ bool decode_rounds(const DecodeArgs &a, const ChunkOut<KV> &geo, const uint32_t *src,
                                              bool ok, uint32_t nc, uint32_t nr, uint32_t nu,
                                              const uint32_t *startbit, const uint32_t *sign_tab,
                                              const float *rot_s, int r0, int r1, int lane) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    const int k = KC >= 0 ? KC : a.k, kl = KC >= 0 ? KC : a.k_last;
    const int q = lane & 3;
    const uint32_t *un = src + nc + nr;
    const float2 e2 = make_float2(geo.e_scale, geo.e_scale);
    const uint32_t pk = 1u << k, pkl = 1u << kl;   // quotient weights 2^k, and 2^kl of a block's last symbol
    const uint32_t gbits = group_rem_bits<N>(k, kl), lane_bits = 4u * gbits;
    bool bad = false;
    const int nrounds = min((geo.ntiles + kTilesPerRound - 1) / kTilesPerRound, r1);
#pragma unroll 1
    for (int r = r0; r < nrounds; r++) {
        char *dst = nullptr;
        int tcol = 0;
        unsigned long long e0 = 0;
        long long pos = -1;
        const bool valid = geo.template tile<MODE>(a, r * kTilesPerRound + (lane >> 2), dst, tcol, e0, pos);
        const uint32_t segi = 32u * r + lane;
        float2 v[16];
        bool lane_ok = ok;
        if (ok && valid) {
            uint32_t bp = startbit[segi];
            const uint32_t *rw = src + nc + segi * (uint32_t)k;
            uint32_t rx[4] = {0u, 0u, 0u, 0u};
            if (KSMALL && k > 0) rem_windows(rw, k, rx);
            const uint32_t cw = (LAT == HQ_E8) ? src[4 * r + (lane >> 3)] : 0u;
            const uint32_t coset = (cw >> (4 * (lane & 7))) & 0xFu;
            const unsigned long long eq = e0 + 32ull * q;
#pragma unroll
            for (int g = 0; g < 4; g++) {
                uint32_t qv[8], rv[8];
                unary4<STAGED>(un, nu, bp, lane_ok, qv);
                unary4<STAGED>(un, nu, bp, lane_ok, qv + 4);
                if (KSMALL) {
                    const uint32_t mask = (1u << k) - 1u;
                    uint32_t xw = rx[g];
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        rv[i] = xw & mask;
                        xw >>= k;
                    }
                } else {
                    if (MIXED)
                        rem_group_mixed<N, STAGED>(src + nc, nr, segi * lane_bits, g, k, kl, gbits, rv);
                    else
                        rem_group(rw, k, g, rv);
                }
                float u[8];
#pragma unroll
                for (int bb = 0; bb < 8 / N; bb++) {
                    const int b = g * (8 / N) + bb;
                    int32_t qq[N];
                    float p[N];
                    if constexpr (LAT == HQ_E8) {
                        uint32_t zb[8];
#pragma unroll
                        for (int i = 0; i < 8; i++) zb[i] = imad(qv[bb * N + i], i == N - 1 ? pkl : pk, rv[bb * N + i]);
                        e8_codes_from_symbols(zb, (coset >> b) & 1u, qq);
                    } else {
                        int32_t m[N];
#pragma unroll
                        for (int i = 0; i < N; i++)
                            m[i] = unzigzag(imad(qv[bb * N + i], (N > 1 && i == N - 1) ? pkl : pk, rv[bb * N + i]));
                        L::reinsert(m, (coset >> b) & 1u, qq);
                    }
                    decoded_point<LAT>(qq, p);
                    if (DITHER) {
                        float d[N];
                        dither_block<LAT>(a.seed, eq + (unsigned long long)(8 * g + bb * N), d);
#pragma unroll
                        for (int i = 0; i < N; i++) p[i] = __fsub_rn(p[i], d[i]);
                    }
#pragma unroll
                    for (int i = 0; i < N; i++) u[bb * N + i] = p[i];
                }
#pragma unroll
                for (int j = 0; j < 4; j++) v[4 * g + j] = f2_mul(make_float2(u[2 * j], u[2 * j + 1]), e2);
            }
            if (bp > nu * 32u) lane_ok = false;
        } else {
#pragma unroll
            for (int j = 0; j < 16; j++) v[j] = make_float2(0.0f, 0.0f);
        }
        if (valid && !lane_ok) bad = true;
        if constexpr (ROT) {
            rotate_round(v, rot_s, lane);
        } else {
            fwht128_quarter(v, lane);
        }
        // a tile is written as zeros unless all four of its lanes decoded
        const unsigned bad_lanes = __ballot_sync(0xffffffffu, valid && !lane_ok);
        const bool tile_bad = (bad_lanes >> (lane & ~3)) & 0xFu;
        if constexpr (MODE == kGemvPartials || MODE == kKvScores) {
            // the tile as hq_dequantize stores it in bf16, then dot products with the vector(s)
            const uint32_t es = ROT ? 0u : sign_tab[tcol * kSignWords + q];
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; j++) {
                __nv_bfloat162 hb = __floats2bfloat162_rn(v[j].x, v[j].y);
                w[j] = tile_bad ? 0u : (*reinterpret_cast<uint32_t *>(&hb) ^ sign_pair_mask(es, j));
            }
            if constexpr (MODE == kGemvPartials) {
                const float acc = tile_sum(valid ? lane_dot(w, a.vec + (long long)tcol * kTile + 32 * q) : 0.0f);
                if (valid && q == 0) a.res[pos] = acc;
            } else {
                // every query head of the KV head's group; a tile past len (pos < 0) only joins the shuffles
                for (int gq = 0; gq < a.group; gq++) {
                    const long long qh = geo.h * a.group + gq;
                    const float acc = tile_sum(pos >= 0 ? lane_dot(w, a.vec + qh * kTile + 32 * q) : 0.0f);
                    if (pos >= 0 && q == 0) a.res[qh * a.out_ld + pos] = acc;
                }
            }
        } else if (dst) {
            // a bad tile is stored as +0: its values zeroed and no sign flipped (rare, so a
            // branch rather than a select per word)
            uint32_t es = ROT ? 0u : sign_tab[tcol * kSignWords + q];
            if (tile_bad) {
                es = 0u;
#pragma unroll
                for (int j = 0; j < 16; j++) v[j] = make_float2(0.0f, 0.0f);
            }
            if (MODE != kStoreBf16 && a.out_fp32) {
                uint4 *o = reinterpret_cast<uint4 *>(dst) + 8 * q;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint32_t m0 = sign_pair_mask(es, 2 * j), m1 = sign_pair_mask(es, 2 * j + 1);
                    uint4 w;
                    w.x = __float_as_uint(v[2 * j].x) ^ (m0 << 16);
                    w.y = __float_as_uint(v[2 * j].y) ^ (m0 & 0x80000000u);
                    w.z = __float_as_uint(v[2 * j + 1].x) ^ (m1 << 16);
                    w.w = __float_as_uint(v[2 * j + 1].y) ^ (m1 & 0x80000000u);
                    o[j] = w;
                }
            } else {
                uint4 *o = reinterpret_cast<uint4 *>(dst) + 4 * q;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t pk[4];
#pragma unroll
                    for (int u2 = 0; u2 < 4; u2++) {
                        __nv_bfloat162 hb = __floats2bfloat162_rn(v[4 * j + u2].x, v[4 * j + u2].y);
                        pk[u2] = *reinterpret_cast<uint32_t *>(&hb) ^ sign_pair_mask(es, 4 * j + u2);
                    }
                    o[j] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }
    return bad;
}

// Three CTAs (24 warps) per SM without dither, where the decoder fits 80 registers with
// almost no spills; two with dither, whose second lattice search needs more; with the
// dense rotation one CTA of kRotDecodeWarps warps, whose shared form of Q^T and per-warp
// rotation buffers (rot_smem_bytes) come first.
// MIXED: the last symbol of each block has its own Rice parameter (a.k_last != a.k).
// KC >= 0: the Rice parameter is KC (= a.k = a.k_last), fixed at compile time.
template <int LAT, bool DITHER, bool KV, bool KSMALL, int MODE, bool ROT = false, bool MIXED = false, int KC = -1>
__global__ void __launch_bounds__((ROT ? kRotDecodeWarps : kWarpsPerCta) * 32, ROT ? 1 : ((DITHER || MIXED) ? 2 : 3))
    decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int kStageSlot = kStageWords + kStagePad;
    constexpr int W = ROT ? kRotDecodeWarps : kWarpsPerCta;
    const float *rot_s = ROT ? reinterpret_cast<const float *>(smem) : nullptr;
    uint32_t *sign_tab = smem + (ROT ? rot_smem_bytes(W) / sizeof(uint32_t) : 0);
    uint32_t *stage_all = sign_tab + a.tcols * kSignWords;
    uint32_t *start_all = stage_all + W * 2 * kStageSlot;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *stages = stage_all + warp * 2 * kStageSlot;
    uint32_t *startbit = start_all + warp * 128;   // first unary bit of every 32-symbol segment

    if (ROT)
        load_rotation<false>(reinterpret_cast<float *>(smem), a.rot);
    else
        build_sign_table(sign_tab, a.tcols, a.seed);
    __syncthreads();

    const int k = KC >= 0 ? KC : a.k;
    uint32_t status = 0;
    // Which rounds this warp decodes: m = 2^lg = 1, 2 or 4 warps share a chunk, 4 / m
    // rounds each, with m as large as the launch's chunks leave warps for.  The warp's
    // slices are v = gw, gw + nwarps, ... (one when m > 1): chunk v / m, rounds from
    // (v mod m) * 4 / m.  Warps are numbered across CTAs first when m > 1 (always in the
    // rotation decoder), so that a short launch spreads over every SM.
    const unsigned long long nwarps = (unsigned long long)gridDim.x * W;
    const int lg = 4 * a.n_chunks <= nwarps ? 2 : 2 * a.n_chunks <= nwarps ? 1 : 0;
    unsigned long long v = (ROT || lg) ? (unsigned long long)warp * gridDim.x + blockIdx.x
                                       : (unsigned long long)blockIdx.x * W + warp;
    int buf = 0;
    ChunkWords cw = {0, 0, false, nullptr, 0, 0};
    if ((v >> lg) < a.n_chunks) {
        cw = chunk_words(a, v >> lg);
        stage_chunk(a, cw, stages, lane);
    }
    for (; (v >> lg) < a.n_chunks; v += nwarps, buf ^= 1) {
        // start bringing in the next chunk while this one is decoded
        const unsigned long long cn = (v + nwarps) >> lg;
        ChunkWords cwn = {0, 0, false, nullptr, 0, 0};
        if (cn < a.n_chunks) {
            cwn = chunk_words(a, cn);
            stage_chunk(a, cwn, stages + (buf ^ 1) * kStageSlot, lane);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();

        const int r0 = (int)(v & ((1u << lg) - 1u)) << (2 - lg), r1 = r0 + (kRoundsPerChunk >> lg);
        ChunkOut<KV> geo;
        geo.init(a, cw.local, cw.item);
        const int ntiles = geo.ntiles;
        const uint32_t nsym = (uint32_t)ntiles * kTile, nseg = 4u * (uint32_t)ntiles;
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
        const uint32_t nr = ((uint32_t)ntiles * tile_rem_bits<Lattice<LAT>::N>(k, a.k_last) + 31u) >> 5;
        bool ok = cw.ok && cw.nw >= (unsigned long long)(nc + nr) &&
                  (cw.nw - nc - nr) < (unsigned long long)(kMaxUnaryBits / 32u);
        const bool staged = cw.nw <= (unsigned long long)kStageWords;
        const uint32_t nu = ok ? (uint32_t)(cw.nw - nc - nr) : 0u;
        // the staged and in-place paths get distinct pointer expressions so the
        // staged one keeps its shared-memory address space after inlining
        bool bad;
        if (staged) {
            const uint32_t *src = stages + buf * kStageSlot;
            ok = find_segment_starts(src + nc + nr, nu, nsym, nseg, ok, startbit, lane);
            bad = decode_rounds<LAT, DITHER, KV, KSMALL, true, MODE, ROT, MIXED, KC>(a, geo, src, ok, nc, nr, nu, startbit, sign_tab,
                                                                          rot_s, r0, r1, lane);
        } else {
            const uint32_t *src = cw.src;
            ok = find_segment_starts(src + nc + nr, nu, nsym, nseg, ok, startbit, lane);
            bad = decode_rounds<LAT, DITHER, KV, KSMALL, false, MODE, ROT, MIXED, KC>(a, geo, src, ok, nc, nr, nu, startbit,
                                                                           sign_tab, rot_s, r0, r1, lane);
        }
        if (__any_sync(0xffffffffu, bad || (!ok && ntiles > 0))) {
            if (a.batch > 1) {
                if (lane == 0 && a.stats) atomicOr(&a.stats[cw.item].status, HQ_ST_CORRUPT);
            } else {
                status |= HQ_ST_CORRUPT;
            }
        }
        cw = cwn;
        __syncwarp();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (a.stats) {
        status = __reduce_or_sync(0xffffffffu, status);
        if (lane == 0 && status) atomicOr(&a.stats->status, status);
    }
}

}  // namespace
}  // namespace hq
