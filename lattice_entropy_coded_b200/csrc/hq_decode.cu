// hq_decode.cu -- decode + dequantize kernel (HyperQuant "Methodology" sections
// 1-4 inverted): Rice planes -> symbols -> re-inserted membership bits ->
// lattice point [- dither] -> scale -> FWHT-128 -> sign -> bf16 (or fp32).
//
// Work decomposition (B200, sm_100a): one warp decodes one chunk, one lane owns
// one tile.  The chunk's words are staged in shared memory with coalesced
// loads; the lanes split the unary plane into 32 segments, count terminators
// (popc) and scan, so every lane learns where its tile's first codeword starts;
// then each lane decodes its 128 quotients sequentially from a bit-reversed
// 32-bit window (one count-leading-zeros and one shift per symbol), pulls the k
// remainder bits from its own fixed region, and runs the inverse transform in
// registers.  Chunks are independent (offsets are given), so no look-back.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq_device.cuh"

namespace hq {

namespace {

// 32 bits of a plane of `n` words starting at bit `b` (bits past the plane are 0).
__device__ __forceinline__ uint32_t fetch32(const uint32_t *p, uint32_t n, uint32_t b) {
    uint32_t w = b >> 5;
    uint32_t a0 = (w < n) ? p[w] : 0u;
    uint32_t a1 = (w + 1 < n) ? p[w + 1] : 0u;
    return __funnelshift_r(a0, a1, b & 31u);
}

// Sequential reader of one lane's unary quotients: a bit-reversed 32-bit
// window, so a quotient is one count-leading-zeros and one shift.  Groups of 8
// whose codes fit in the window take the fast path; longer ones go bit-word by
// bit-word.  `ok` turns false if the plane ends early.
struct UnaryReader {
    const uint32_t *un;
    uint32_t nu, nbits, bp;
    bool ok;

    __device__ __forceinline__ void init(const uint32_t *p, uint32_t n, uint32_t start) {
        un = p;
        nu = n;
        nbits = n * 32u;
        bp = start;
        ok = true;
    }
    __device__ __forceinline__ void group(uint32_t (&q)[8]) {
        uint32_t w = __brev(fetch32(un, nu, bp));   // next 32 stream bits, first at the MSB
        if (__popc(w) >= 8) {
            uint32_t used = 8;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                uint32_t t = __clz(w);
                q[i] = t;
                used += t;
                w = (w << t) << 1;
            }
            bp += used;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) {
                uint32_t t = 0;
                uint32_t x = __brev(fetch32(un, nu, bp));
                while (x == 0u && ok) {
                    t += 32u;
                    bp += 32u;
                    if (bp >= nbits) ok = false;
                    x = __brev(fetch32(un, nu, bp));
                }
                uint32_t c = __clz(x);
                t += c;
                bp += c + 1u;
                q[i] = t;
            }
        }
        if (bp > nbits) ok = false;
    }
};

// k-bit remainders of one group of 8 symbols from the lane's region `rw` (4k words).
__device__ __forceinline__ void rem_group(const uint32_t *rw, int k, int g, uint32_t (&r)[8]) {
    if (k == 0) {
#pragma unroll
        for (int i = 0; i < 8; i++) r[i] = 0;
        return;
    }
    const uint32_t n = 4u * (uint32_t)k;
    const uint32_t mask = (1u << k) - 1u;
    const uint32_t b = (uint32_t)(8 * g) * (uint32_t)k;
    if (k <= 4) {
        uint32_t x = fetch32(rw, n, b);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            r[i] = x & mask;
            x >>= k;
        }
    } else if (k <= 8) {
        unsigned long long x = ((unsigned long long)fetch32(rw, n, b + 32u) << 32) | fetch32(rw, n, b);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            r[i] = (uint32_t)x & mask;
            x >>= k;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) r[i] = fetch32(rw, n, b + (uint32_t)(i * k)) & mask;
    }
}

struct TileOut {
    bool valid;
    char *dst;          // first element of the tile in `out`
    int tcol;
    unsigned long long e0;
    float e_scale;
};

template <bool KV>
__device__ __forceinline__ void tile_out(const DecodeArgs &a, unsigned long long c, int lane, TileOut &t,
                                         int &ntiles) {
    const size_t esz = a.out_fp32 ? 4 : 2;
    if (KV) {
        // the append that holds global chunk c (binary search on first_chunk)
        unsigned long long lo = 0, hi = a.n_appends - 1;
        while (lo < hi) {
            unsigned long long mid = (lo + hi + 1) >> 1;
            if (a.table[mid].first_chunk <= c) lo = mid; else hi = mid - 1;
        }
        const hq_kv_append_row row = a.table[lo];
        long long T = row.tokens;
        long long cph = (T + 31) / 32;
        long long lc = (long long)(c - row.first_chunk);
        long long h = lc / cph, tc = lc % cph;
        long long tok = tc * 32 + lane;
        long long ntok = T - tc * 32;
        ntiles = (int)(ntok < 32 ? ntok : 32);
        long long gt = row.token0 + tok;
        t.valid = tok < T;
        t.e_scale = row.scale_inv;
        t.tcol = 0;
        t.e0 = (unsigned long long)((gt * a.map.heads + h) * kTile);
        t.dst = (t.valid && gt < a.len) ? (char *)a.out + (size_t)(h * a.out_ld_head + gt * a.out_ld) * esz : nullptr;
        return;
    }
    long long tpr = a.map.cols / kTile;
    long long ntile_all = a.map.rows * tpr;
    long long t0 = (long long)c * 32;
    long long ti = t0 + lane;
    ntiles = (int)((ntile_all - t0) < 32 ? (ntile_all - t0) : 32);
    t.valid = ti < ntile_all;
    long long r = ti / tpr, tc = ti % tpr;
    t.tcol = (int)tc;
    t.e0 = (unsigned long long)(r * a.map.cols + tc * kTile);
    t.e_scale = a.e_scale;
    t.dst = t.valid ? (char *)a.out + (size_t)(r * a.out_ld + tc * kTile) * esz : nullptr;
}

template <int LAT, bool DITHER, bool KV>
__global__ void __launch_bounds__(kWarpsPerCta * 32, 1) decode_kernel(const DecodeArgs a) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *sign_tab = smem;
    uint32_t *rows_all = smem + a.tcols * kSignStride;
    uint32_t *stage_all = rows_all + kWarpsPerCta * 32 * kRowStride;
    uint32_t *start_all = stage_all + kWarpsPerCta * kStageWords;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *row = reinterpret_cast<float *>(rows_all + (warp * 32 + lane) * kRowStride);
    uint32_t *stage = stage_all + warp * kStageWords;
    uint32_t *startbit = start_all + warp * 32;

    for (int i = threadIdx.x; i < a.tcols * 64; i += blockDim.x) {
        int tc = i >> 6, p = i & 63;
        unsigned long long col = (unsigned long long)tc * kTile + 2 * p;
        sign_tab[tc * kSignStride + p] = (sign_bit(a.seed, col) << 15) | (sign_bit(a.seed, col + 1) << 31);
    }
    __syncthreads();

    const int k = a.k;
    uint32_t status = 0;
    const unsigned long long nwarps = (unsigned long long)gridDim.x * kWarpsPerCta;
    for (unsigned long long c = (unsigned long long)blockIdx.x * kWarpsPerCta + warp; c < a.n_chunks; c += nwarps) {
        TileOut t;
        int ntiles = 0;
        tile_out<KV>(a, c, lane, t, ntiles);
        const unsigned long long w0 = a.offsets[c], w1 = a.offsets[c + 1];
        const uint32_t nsym = (uint32_t)ntiles * kTile;
        const unsigned long long nc = (LAT == HQ_E8) ? (unsigned long long)(16 * ntiles + 31) / 32 : 0ull;
        const unsigned long long nr = 4ull * (unsigned long long)k * (unsigned long long)ntiles;
        bool ok = w0 <= w1 && w1 <= a.stream_words && (w1 - w0) >= nc + nr &&
                  (w1 - w0 - nc - nr) < (unsigned long long)(kMaxUnaryBits / 32u);
        const unsigned long long nw = ok ? w1 - w0 : 0ull;
        const bool staged = nw <= (unsigned long long)kStageWords;
        const uint32_t *src = staged ? stage : a.stream + w0;
        if (staged) {
            for (unsigned long long i = lane; i < nw; i += 32) stage[i] = __ldg(a.stream + w0 + i);
        }
        __syncwarp();
        const uint32_t nu = ok ? (uint32_t)(nw - nc - nr) : 0u;
        const uint32_t *un = src + nc + nr;

        // ---- where does each tile's first codeword start?  (popc + scan over 32 segments)
        const uint32_t seg = (nu + 31u) / 32u;
        const uint32_t s0 = min(nu, (uint32_t)lane * seg), s1 = min(nu, s0 + seg);
        uint32_t cnt = 0;
        for (uint32_t i = s0; i < s1; i++) cnt += __popc(un[i]);
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const uint32_t ones = __shfl_sync(0xffffffffu, incl, 31);
        ok = ok && ones == nsym;
        if (ok) {
            const uint32_t before = incl - cnt;
            // terminator index j = 128 t - 1 of tile t = 1..ntiles-1 inside [before, incl)
            uint32_t tt = (before + 1u + 127u) / 128u;
            if (tt == 0) tt = 1;
            uint32_t i = s0, seen = before;
            for (; tt < (uint32_t)ntiles && 128u * tt - 1u < incl; tt++) {
                const uint32_t j = 128u * tt - 1u;
                uint32_t w = un[i], pc = __popc(w);
                while (seen + pc <= j) {
                    seen += pc;
                    i++;
                    w = un[i];
                    pc = __popc(w);
                }
                for (uint32_t r = j - seen; r; r--) w &= w - 1u;   // drop the lower set bits
                startbit[tt] = i * 32u + (uint32_t)(__ffs(w) - 1) + 1u;
            }
            if (lane == 0) startbit[0] = 0;
        }
        __syncwarp();

        // ---- symbols -> lattice points -> scaled coordinates, group by group into the row
        bool lane_ok = ok;
        if (ok && t.valid) {
            UnaryReader ur;
            ur.init(un, nu, startbit[lane]);
            const uint32_t *rw = src + nc + 4ull * k * lane;
            const uint32_t coset = (LAT == HQ_E8) ? (src[lane >> 1] >> (16 * (lane & 1))) & 0xFFFFu : 0u;
#pragma unroll 1
            for (int g = 0; g < kTile / 8; g++) {
                uint32_t qv[8], rv[8];
                ur.group(qv);
                rem_group(rw, k, g, rv);
                float u[8];
#pragma unroll
                for (int bb = 0; bb < 8 / N; bb++) {
                    const int b = g * (8 / N) + bb;
                    int32_t m[N], q[N];
                    float p[N];
#pragma unroll
                    for (int i = 0; i < N; i++) m[i] = unzigzag((qv[bb * N + i] << k) | rv[bb * N + i]);
                    L::reinsert(m, (coset >> b) & 1u, q);
                    L::point(q, p);
                    if (DITHER) {
                        float d[N];
                        dither_block<LAT>(a.seed, t.e0 + (unsigned long long)(8 * g + bb * N), d);
#pragma unroll
                        for (int i = 0; i < N; i++) p[i] = __fsub_rn(p[i], d[i]);
                    }
#pragma unroll
                    for (int i = 0; i < N; i++) u[bb * N + i] = p[i];
                }
                const float2 e2 = make_float2(t.e_scale, t.e_scale);
                float2 s0v = f2_mul(make_float2(u[0], u[1]), e2), s1v = f2_mul(make_float2(u[2], u[3]), e2);
                float2 s2v = f2_mul(make_float2(u[4], u[5]), e2), s3v = f2_mul(make_float2(u[6], u[7]), e2);
                *reinterpret_cast<float4 *>(row + 8 * g) = make_float4(s0v.x, s0v.y, s1v.x, s1v.y);
                *reinterpret_cast<float4 *>(row + 8 * g + 4) = make_float4(s2v.x, s2v.y, s3v.x, s3v.y);
            }
            lane_ok = ur.ok;
        }
        if (__any_sync(0xffffffffu, t.valid && !(ok && lane_ok))) status |= HQ_ST_CORRUPT;

        // ---- FWHT, sign, round, store
        if (t.dst) {
            const bool good = ok && lane_ok;
            float2 v[kTile / 2];
#pragma unroll
            for (int j = 0; j < kTile / 4; j++) {
                float4 f = good ? *reinterpret_cast<const float4 *>(row + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[2 * j] = make_float2(f.x, f.y);
                v[2 * j + 1] = make_float2(f.z, f.w);
            }
            fwht128(v);
            const uint32_t *sg = sign_tab + t.tcol * kSignStride;
            if (a.out_fp32) {
                uint4 *o = reinterpret_cast<uint4 *>(t.dst);
#pragma unroll
                for (int j = 0; j < kTile / 4; j++) {
                    const uint32_t s0w = sg[2 * j], s1w = sg[2 * j + 1];
                    uint4 w;
                    w.x = __float_as_uint(v[2 * j].x) ^ (s0w << 16);
                    w.y = __float_as_uint(v[2 * j].y) ^ (s0w & 0x80000000u);
                    w.z = __float_as_uint(v[2 * j + 1].x) ^ (s1w << 16);
                    w.w = __float_as_uint(v[2 * j + 1].y) ^ (s1w & 0x80000000u);
                    o[j] = w;
                }
            } else {
                uint4 *o = reinterpret_cast<uint4 *>(t.dst);
#pragma unroll
                for (int j = 0; j < kTile / 8; j++) {
                    const uint4 s = *reinterpret_cast<const uint4 *>(sg + 4 * j);
                    const uint32_t sw[4] = {s.x, s.y, s.z, s.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int u2 = 0; u2 < 4; u2++) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[4 * j + u2].x, v[4 * j + u2].y);
                        pk[u2] = *reinterpret_cast<uint32_t *>(&h) ^ sw[u2];
                    }
                    o[j] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
        __syncwarp();
    }
    if (a.stats) {
        status = __reduce_or_sync(0xffffffffu, status);
        if (lane == 0 && status) atomicOr(&a.stats->status, status);
    }
}

template <int LAT, bool DITHER, bool KV>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(a.tcols * kSignStride + kWarpsPerCta * 32 * kRowStride + kWarpsPerCta * kStageWords +
                                 kWarpsPerCta * 32) *
                        sizeof(uint32_t);
    auto kern = decode_kernel<LAT, DITHER, KV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpsPerCta * 32, smem)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    unsigned long long want = (a.n_chunks + kWarpsPerCta - 1) / kWarpsPerCta;
    unsigned long long grid = (unsigned long long)sms * (unsigned long long)per_sm;
    if (want < grid) grid = want;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, kWarpsPerCta * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool KV>
cudaError_t dispatch(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_t<HQ_Z, false, KV>(a, s);
    case HQ_Z * 2 + 1: return launch_t<HQ_Z, true, KV>(a, s);
    case HQ_A2 * 2: return launch_t<HQ_A2, false, KV>(a, s);
    case HQ_A2 * 2 + 1: return launch_t<HQ_A2, true, KV>(a, s);
    case HQ_D4 * 2: return launch_t<HQ_D4, false, KV>(a, s);
    case HQ_D4 * 2 + 1: return launch_t<HQ_D4, true, KV>(a, s);
    case HQ_E8 * 2: return launch_t<HQ_E8, false, KV>(a, s);
    case HQ_E8 * 2 + 1: return launch_t<HQ_E8, true, KV>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(int lattice, int dither, const DecodeArgs &a, cudaStream_t s) {
    return a.map.kv ? dispatch<true>(lattice, dither, a, s) : dispatch<false>(lattice, dither, a, s);
}

}  // namespace hq
