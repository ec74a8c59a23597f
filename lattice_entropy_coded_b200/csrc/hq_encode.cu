// hq_encode.cu -- quantize + encode kernel (HyperQuant "Methodology" sections
// 1-4): per 128-element tile, seeded sign flip, FWHT-128, scale, optional
// subtractive dither, nearest lattice point, bit-stripping, zigzag, Rice planes.
//
// Work decomposition (B200, sm_100a):
//  * one warp encodes one chunk (32 tiles), one lane owns one tile: load, sign
//    flip, FWHT and scale run on 64 float2 registers with packed fp32 adds;
//  * the transformed tile goes to a lane-private shared-memory row, and pass A
//    walks it in a rolled loop over groups of 8 coordinates (one copy of the
//    lattice decoder in the instruction stream), leaving the zigzag symbols in
//    the row in place;
//  * a persistent grid; warps take chunk tickets from a global counter, so a
//    chunk's predecessors are always already running;
//  * warp scan of the unary lengths and a single-pass decoupled look-back over
//    64-bit (flag, value) words give the chunk's word offset (bounded waits:
//    HQ_ST_TIMEOUT);
//  * pass B builds the remainder and unary planes in a per-warp shared stage
//    and writes the chunk with coalesced stores; a chunk larger than the stage,
//    or with quotients above 255, is written in place in global memory.
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

// Exclusive prefix (in words) of chunk c over chunks [0, c) of this call.
// Whole warp calls it; lane 0 publishes.  Bounded: gives up after spin_limit polls.
__device__ __noinline__ unsigned long long lookback(unsigned long long *lb, unsigned long long c,
                                                    unsigned long long agg, uint32_t spin_limit, bool &timed_out) {
    const int lane = threadIdx.x & 31;
    if (c == 0) {
        if (lane == 0) st_relaxed_u64(lb, kFlagInc | agg);
        return 0;
    }
    if (lane == 0) st_relaxed_u64(lb + c, kFlagAgg | agg);
    unsigned long long excl = 0;
    long long pos = (long long)c - 1;
    uint32_t spins = 0;
    while (true) {
        long long idx = pos - lane;
        unsigned long long v = (idx >= 0) ? ld_relaxed_u64(lb + idx) : kFlagInc;
        unsigned flag = (unsigned)(v >> 62);
        unsigned inc = __ballot_sync(0xffffffffu, flag == 2u);
        unsigned zero = __ballot_sync(0xffffffffu, flag == 0u);
        int first_inc = inc ? __ffs(inc) - 1 : 32;
        unsigned relevant = (first_inc >= 31) ? 0xffffffffu : ((2u << first_inc) - 1u);
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

// Tile of lane `lane` in chunk c: source pointer, sign-table column, dither counter.
__device__ __forceinline__ bool tile_of(const TileMap &m, const uint16_t *x, unsigned long long c, int lane,
                                        const uint16_t *&src, int &tcol, unsigned long long &e0, int &ntiles) {
    if (m.kv) {
        long long cph = (m.tokens + 31) / 32;
        long long h = (long long)c / cph, tc = (long long)c % cph;
        long long tok = tc * 32 + lane;
        long long left = m.tokens - tc * 32;
        ntiles = (int)(left < 32 ? left : 32);
        if (tok >= m.tokens) return false;
        src = x + h * m.ld_head + tok * m.ld_tok;
        tcol = 0;
        e0 = (unsigned long long)(((m.tok0 + tok) * m.heads + h) * kTile);
        return true;
    }
    long long tpr = m.cols / kTile;
    long long all = m.rows * tpr;
    long long t0 = (long long)c * 32;
    ntiles = (int)((all - t0) < 32 ? (all - t0) : 32);
    long long t = t0 + lane;
    if (t >= all) return false;
    long long r = t / tpr, tc = t % tpr;
    src = x + r * m.ld + tc * kTile;
    tcol = (int)tc;
    e0 = (unsigned long long)(r * m.cols + tc * kTile);
    return true;
}

// x (bf16, 128 elements) -> D x widened to fp32 -> H_128 -> * c, stored to the
// lane's row (16-byte stores).
__device__ __forceinline__ void transform_to_row(const uint16_t *src, bool valid, const uint32_t *sg, float c_scale,
                                                 float *row) {
    float2 v[kTile / 2];
#pragma unroll
    for (int j = 0; j < kTile / 8; j++) {
        uint4 w = valid ? ldg_nc_v4(src + 8 * j) : make_uint4(0, 0, 0, 0);
        uint4 s = *reinterpret_cast<const uint4 *>(sg + 4 * j);
        uint32_t ww[4] = {w.x ^ s.x, w.y ^ s.y, w.z ^ s.z, w.w ^ s.w};
#pragma unroll
        for (int t = 0; t < 4; t++)
            v[4 * j + t] = make_float2(__uint_as_float(ww[t] << 16), __uint_as_float(ww[t] & 0xFFFF0000u));
    }
    fwht128(v);
    const float2 c2 = make_float2(c_scale, c_scale);
#pragma unroll
    for (int j = 0; j < kTile / 4; j++) {
        float2 a = f2_mul(v[2 * j], c2), b = f2_mul(v[2 * j + 1], c2);
        *reinterpret_cast<float4 *>(row + 4 * j) = make_float4(a.x, a.y, b.x, b.y);
    }
}

// Symbols of group g (8 coordinates u[0..7]); returns the E8 coset bits of the
// group's blocks (bit bb for block bb of the group).
template <int LAT, bool DITHER>
__device__ __forceinline__ uint32_t group_symbols(const float (&u)[8], int g, unsigned long long e0, uint64_t seed,
                                                  uint32_t (&z)[8]) {
    using L = Lattice<LAT>;
    constexpr int N = L::N;
    uint32_t cb = 0;
#pragma unroll
    for (int bb = 0; bb < 8 / N; bb++) {
        float blk[N];
#pragma unroll
        for (int i = 0; i < N; i++) blk[i] = u[bb * N + i];
        if (DITHER) {
            float d[N];
            dither_block<LAT>(seed, e0 + (unsigned long long)(8 * g + bb * N), d);
#pragma unroll
            for (int i = 0; i < N; i++) blk[i] = __fadd_rn(blk[i], d[i]);
        }
        int32_t q[N], m[N];
        L::nearest(blk, q);
        cb |= L::strip(q, m) << bb;
#pragma unroll
        for (int i = 0; i < N; i++) z[bb * N + i] = zigzag(m[i]);
    }
    return cb;
}

// Remainder plane writer: k low bits per symbol, LSB first, into the lane's own
// region `dst` (4k words).  k is warp-uniform, so the flushes are uniform.
struct RemWriter {
    uint32_t *dst;
    int k;
    uint32_t mask, nb, w;
    bool store;
    unsigned long long acc;

    __device__ __forceinline__ void init(uint32_t *d, int kk, bool st) {
        dst = d;
        k = kk;
        mask = kk ? (1u << kk) - 1u : 0u;
        store = st;
        acc = 0;
        nb = 0;
        w = 0;
    }
    __device__ __forceinline__ void put_group(const uint32_t (&z)[8]) {
        if (k == 0) return;
        if (k <= 4) {
            uint32_t gv = 0;   // 8k <= 32 bits, symbol 0 in the low bits
#pragma unroll
            for (int i = 7; i >= 0; i--) gv = (gv << k) | (z[i] & mask);
            acc |= (unsigned long long)gv << nb;
            nb += 8u * (uint32_t)k;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) {
                acc |= (unsigned long long)(z[i] & mask) << nb;
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
};

// Unary terminators of 8 symbols with quotients q[0..7], starting at bit pos of
// `un` (zeroed words).  A group whose codes fit in 32 bits is built in a
// register (last symbol first) and ORed in with two shared atomics.
__device__ __forceinline__ uint32_t unary_group_shared(uint32_t *un, uint32_t pos, const uint32_t (&q)[8]) {
    uint32_t ug = 8;
#pragma unroll
    for (int i = 0; i < 8; i++) ug += q[i];
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
    return ug;
}

template <int LAT, bool DITHER>
__global__ void __launch_bounds__(kWarpsPerCta * 32, 1) encode_kernel(const EncodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *sign_tab = smem;                                                  // tcols * kSignStride
    uint32_t *rows_all = smem + a.tcols * kSignStride;                          // warps * 32 * kRowStride
    uint32_t *stage_all = rows_all + kWarpsPerCta * 32 * kRowStride;            // warps * kStageWords
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *row = reinterpret_cast<float *>(rows_all + (warp * 32 + lane) * kRowStride);
    uint32_t *zrow = rows_all + (warp * 32 + lane) * kRowStride;
    uint32_t *stage = stage_all + warp * kStageWords;

    // Sign masks per bf16x2 pair: bit 15 flips the even column, bit 31 the odd one.
    for (int i = threadIdx.x; i < a.tcols * 64; i += blockDim.x) {
        int tc = i >> 6, p = i & 63;
        unsigned long long col = (unsigned long long)tc * kTile + 2 * p;
        sign_tab[tc * kSignStride + p] = (sign_bit(a.seed, col) << 15) | (sign_bit(a.seed, col + 1) << 31);
    }
    __syncthreads();

    const int k = a.k;
    const unsigned long long base = a.base_ptr ? *a.base_ptr : 0ull;
    uint32_t status = 0, zor_all = 0;
    unsigned long long payload = 0;

    while (true) {
        unsigned long long c = 0;
        if (lane == 0) c = atomicAdd(a.ticket, 1u);
        c = __shfl_sync(0xffffffffu, c, 0);
        if (c >= a.n_chunks) break;

        const uint16_t *src = nullptr;
        int tcol = 0, ntiles = 0;
        unsigned long long e0 = 0;
        const bool valid = tile_of(a.map, a.x, c, lane, src, tcol, e0, ntiles);
        const uint32_t *sg = sign_tab + tcol * kSignStride;
        transform_to_row(src, valid, sg, a.c_scale, row);

        // ---- pass A: symbols in place of the transformed coordinates
        uint32_t coset = 0, usum = 0, zor = 0;
#pragma unroll 1
        for (int g = 0; g < kTile / 8; g++) {
            const float4 u0 = *reinterpret_cast<const float4 *>(row + 8 * g);
            const float4 u1 = *reinterpret_cast<const float4 *>(row + 8 * g + 4);
            const float u[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t z[8];
            const uint32_t cb = group_symbols<LAT, DITHER>(u, g, e0, a.seed, z);
            coset |= cb << (g * (8 / Lattice<LAT>::N));
#pragma unroll
            for (int i = 0; i < 8; i++) {
                if (!valid) z[i] = 0;
                zor |= z[i];
                usum += z[i] >> k;
            }
            *reinterpret_cast<uint4 *>(zrow + 8 * g) = make_uint4(z[0], z[1], z[2], z[3]);
            *reinterpret_cast<uint4 *>(zrow + 8 * g + 4) = make_uint4(z[4], z[5], z[6], z[7]);
        }
        if (!valid) coset = 0;
        zor_all |= zor;

        // ---- unary lengths: warp scan
        const unsigned long long ubits = valid ? (unsigned long long)usum + kTile : 0ull;
        unsigned long long incl = ubits;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const unsigned long long utotal = __shfl_sync(0xffffffffu, incl, 31);
        const unsigned long long ustart = incl - ubits;
        const uint32_t wzor = __reduce_or_sync(0xffffffffu, zor);
        const bool range_bad = (wzor >> 22) != 0u || utotal >= kMaxUnaryBits;
        if (range_bad) status |= HQ_ST_RANGE;
        const uint32_t nc = (LAT == HQ_E8) ? (uint32_t)(16 * ntiles + 31) / 32u : 0u;
        const uint32_t nr = 4u * (uint32_t)k * (uint32_t)ntiles;
        const unsigned long long nu = (utotal + 31) / 32;
        const unsigned long long total = nc + nr + nu;
        payload += utotal + (unsigned long long)nr * 32 + ((LAT == HQ_E8) ? 16ull * ntiles : 0ull);
        const bool fast = !range_bad && total <= (unsigned long long)kStageWords && (wzor >> (k + 8)) == 0u;

        // ---- chunk offset
        bool to = false;
        const unsigned long long excl = lookback(a.lookback, c, total, a.spin_limit, to);
        if (to) status |= HQ_ST_TIMEOUT;
        const unsigned long long start = base + excl;
        if (lane == 0) {
            a.offsets[a.chunk_base + c] = start;
            if (c + 1 == a.n_chunks) {
                unsigned long long end = start + total;
                a.offsets[a.chunk_base + a.n_chunks] = end;
                if (a.tail_out) *a.tail_out = end;
                if (a.stats) a.stats->stream_words = end;
                if (end > a.cap_words) status |= HQ_ST_CAPACITY;
            }
            if (c == 0 && a.row) *a.row = a.row_val;
        }
        const uint32_t cos_hi = __shfl_down_sync(0xffffffffu, coset, 1);

        if (fast) {
            // ---- pass B: planes into the stage, then one coalesced copy
            for (uint32_t i = nc + nr + lane; i < (uint32_t)total; i += 32) stage[i] = 0u;
            if (LAT == HQ_E8 && (lane & 1) == 0 && (uint32_t)(lane >> 1) < nc) stage[lane >> 1] = coset | (cos_hi << 16);
            __syncwarp();
            RemWriter rw;
            rw.init(stage + nc + 4u * (uint32_t)k * (uint32_t)lane, k, valid);
            uint32_t *un = stage + nc + nr;
            uint32_t pos = (uint32_t)ustart;
#pragma unroll 1
            for (int g = 0; g < kTile / 8; g++) {
                const uint4 z0 = *reinterpret_cast<const uint4 *>(zrow + 8 * g);
                const uint4 z1 = *reinterpret_cast<const uint4 *>(zrow + 8 * g + 4);
                const uint32_t z[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
                rw.put_group(z);
                if (valid) {
                    uint32_t q[8];
#pragma unroll
                    for (int i = 0; i < 8; i++) q[i] = z[i] >> k;
                    pos += unary_group_shared(un, pos, q);
                }
            }
            __syncwarp();
            for (uint32_t i = lane; i < (uint32_t)total; i += 32)
                if (start + i < a.cap_words) a.stream[start + i] = stage[i];
            __syncwarp();
        } else if (!range_bad) {
            // ---- large chunk: zero it in place, then set every bit with a global atomic
            uint32_t *g = a.stream + start;
            const unsigned long long room = (start < a.cap_words) ? a.cap_words - start : 0ull;
            for (unsigned long long i = lane; i < total; i += 32)
                if (i < room) g[i] = 0u;
            __syncwarp();
            __threadfence_block();
            if (LAT == HQ_E8 && (lane & 1) == 0 && (uint32_t)(lane >> 1) < nc && (unsigned long long)(lane >> 1) < room)
                atomicOr(g + (lane >> 1), coset | (cos_hi << 16));
            if (valid) {
                const uint32_t mask = k ? (1u << k) - 1u : 0u;
                unsigned long long rb = 32ull * (nc + 4ull * (unsigned long long)k * lane);
                unsigned long long ub = 32ull * (nc + nr) + ustart;
#pragma unroll 1
                for (int i = 0; i < kTile; i++) {
                    const uint32_t zi = zrow[i];
                    const uint32_t r = zi & mask;
                    for (int b = 0; b < k; b++, rb++)
                        if (((r >> b) & 1u) && (rb >> 5) < room) atomicOr(g + (rb >> 5), 1u << (uint32_t)(rb & 31));
                    ub += zi >> k;
                    if ((ub >> 5) < room) atomicOr(g + (ub >> 5), 1u << (uint32_t)(ub & 31));
                    ub++;
                }
            }
            __syncwarp();
        }
    }

    if (a.stats) {
        zor_all = __reduce_or_sync(0xffffffffu, zor_all);
        status = __reduce_or_sync(0xffffffffu, status);
        if (lane == 0) {
            if (status) atomicOr(&a.stats->status, status);
            if (zor_all) atomicOr(&a.stats->max_symbol, zor_all);
            if (payload) atomicAdd((unsigned long long *)&a.stats->payload_bits, payload);
        }
    }
}

template <int LAT, bool DITHER>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem =
        (size_t)(a.tcols * kSignStride + kWarpsPerCta * 32 * kRowStride + kWarpsPerCta * kStageWords) *
        sizeof(uint32_t);
    auto kern = encode_kernel<LAT, DITHER>;
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

}  // namespace

cudaError_t launch_encode(int lattice, int dither, const EncodeArgs &a, cudaStream_t s) {
    switch (lattice * 2 + (dither ? 1 : 0)) {
    case HQ_Z * 2: return launch_t<HQ_Z, false>(a, s);
    case HQ_Z * 2 + 1: return launch_t<HQ_Z, true>(a, s);
    case HQ_A2 * 2: return launch_t<HQ_A2, false>(a, s);
    case HQ_A2 * 2 + 1: return launch_t<HQ_A2, true>(a, s);
    case HQ_D4 * 2: return launch_t<HQ_D4, false>(a, s);
    case HQ_D4 * 2 + 1: return launch_t<HQ_D4, true>(a, s);
    case HQ_E8 * 2: return launch_t<HQ_E8, false>(a, s);
    case HQ_E8 * 2 + 1: return launch_t<HQ_E8, true>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hq
