// hq_device.cuh -- per-thread device building blocks of the HyperQuant codec:
// counter-based generator, Walsh-Hadamard butterflies, the four lattice
// quantizers in their integer embeddings, bit-stripping and zigzag symbols,
// and the subtractive dither.  One thread owns one 128-element tile in
// registers.  Method: HyperQuant explainer pages, "Methodology" sections 1-4.
//
// Every fp32 operation is an explicit round-to-nearest intrinsic (the file is
// also compiled with --fmad=false), so results are bit-reproducible.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "hq_internal.h"

namespace hq {

// ------------------------------------------------------------------ generator
// SplitMix64 (Steele, Lea & Flood 2014): output number i (0-based) of the
// generator started from state s.  Counter-based: any element's random bits are
// one hash away, so tiles never share generator state.
__device__ __forceinline__ uint64_t splitmix64(uint64_t s, uint64_t i) {
    uint64_t z = s + (i + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// 1 if sign s_j of the RHT diagonal D is -1 (section 1: seeded random signs).
__device__ __forceinline__ uint32_t sign_bit(uint64_t seed, uint64_t j) {
    return (uint32_t)(splitmix64(seed ^ kSignSalt, j) >> 63);
}

// Shared sign table: word 4 tc + q covers columns 128 tc + 32 q + [0, 32): bit t
// (t < 16) is the sign bit of column 2t of the quarter and bit 16 + t that of
// column 2t + 1.  So the XOR mask for the bf16 pair (2t, 2t + 1) held in one
// word (even column in the low half) is sign_pair_mask(E, t): bits 15 and 31.
// Each warp fills words with one generator call per lane and a ballot, lanes
// 0-15 taking the even columns and 16-31 the odd ones.
__device__ __forceinline__ void build_sign_table(uint32_t *tab, int tcols, uint64_t seed) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int off = (lane < 16) ? 2 * lane : 2 * (lane - 16) + 1;
    for (int w = warp; w < tcols * kSignWords; w += nw) {
        const uint32_t e = __ballot_sync(0xffffffffu, sign_bit(seed, (unsigned long long)w * 32ull + off) != 0u);
        if (lane == 0) tab[w] = e;
    }
}
__device__ __forceinline__ uint32_t sign_pair_mask(uint32_t e, int t) { return (e << (15 - t)) & 0x80008000u; }

// ------------------------------------------------------------------ packed fp32
// sm_100 executes two IEEE round-to-nearest fp32 operations per instruction on
// a register pair (add/sub/mul .rn.f32x2); each lane is rounded exactly like the
// scalar operation, so results are bit-identical to scalar code.
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long *>(&a)),
        "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return *reinterpret_cast<float2 *>(&r);
}
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long *>(&a)),
        "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return *reinterpret_cast<float2 *>(&r);
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long *>(&a)),
        "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return *reinterpret_cast<float2 *>(&r);
}

__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(*reinterpret_cast<unsigned long long *>(&a)),
        "l"(*reinterpret_cast<unsigned long long *>(&b)), "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&r);
}

// ------------------------------------------------------------------ FWHT-128 on 4 lanes
// Unnormalised Walsh-Hadamard transform in Sylvester order, radix-2 stages
// h = 1, 2, ..., 64, pair (i, i + h) -> (a + b, a - b).  Four consecutive lanes
// hold one tile, lane quarter q = lane & 3 holding elements [32q, 32q + 32) as
// 16 float2.  Stages 1..16 are inside a lane (stage 1 inside each float2, the
// others with packed adds); stage 32 pairs quarters q and q ^ 1, stage 64 q and
// q ^ 2: the partner's values arrive by shuffle and the lower quarter keeps
// a + b = fma(+1, x, y), the upper a - b = fma(-1, x, y) (exact product, one
// rounding: identical to the subtraction).  The 1/sqrt(128) of the orthonormal
// H_128 is folded into the scale factors.
__device__ __forceinline__ void fwht128_quarter(float2 (&v)[16], int lane) {
#pragma unroll
    for (int j = 0; j < 16; j++) {
        float a = v[j].x, b = v[j].y;
        v[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < 16; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 16; j++) {
            if ((j & hp) == 0) {
                float2 a = v[j], b = v[j + hp];
                v[j] = f2_add(a, b);
                v[j + hp] = f2_sub(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
        const float sg = (lane & m) ? -1.0f : 1.0f;
        const float2 s2 = make_float2(sg, sg);
#pragma unroll
        for (int j = 0; j < 16; j++) {
            float2 y;
            y.x = __shfl_xor_sync(0xffffffffu, v[j].x, m);
            y.y = __shfl_xor_sync(0xffffffffu, v[j].y, m);
            v[j] = f2_fma(s2, v[j], y);
        }
    }
}

// The same transform with sixteen lanes per tile (two tiles per warp): lane l of
// its half-warp holds elements [8l, 8l + 8) as 4 float2.  Stages 1, 2, 4 are inside
// the lane (stage 1 inside each float2, 2 and 4 packed); stages 8, 16, 32, 64 pair
// lane l with l ^ 1, 2, 4, 8 by shuffle, with the same exact fma(+-1, x, y).  The
// butterflies and their order are those of fwht128_quarter, element for element.
__device__ __forceinline__ void fwht128_sixteenth(float2 (&v)[4], int lane) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float a = v[j].x, b = v[j].y;
        v[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < 4; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if ((j & hp) == 0) {
                const float2 a = v[j], b = v[j + hp];
                v[j] = f2_add(a, b);
                v[j + hp] = f2_sub(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m <= 8; m <<= 1) {
        const float sg = (lane & m) ? -1.0f : 1.0f;
        const float2 s2 = make_float2(sg, sg);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            float2 y;
            y.x = __shfl_xor_sync(0xffffffffu, v[j].x, m);
            y.y = __shfl_xor_sync(0xffffffffu, v[j].y, m);
            v[j] = f2_fma(s2, v[j], y);
        }
    }
}

// ------------------------------------------------------------------ dense rotation (KV)
// The KV path may rotate each token's head vector by a full 128 x 128 orthogonal
// matrix Q (a Haar-uniform draw) instead of the sign diagonal and H_128 (explainer
// pages, "Methodology" 4).  Forward y = Q x, inverse x = Q^T z; each output is one
// fp32 fma per term in increasing input index from +0.
//
// rotate_round applies a matrix M to the eight tiles a warp holds in the FWHT's
// quarter layout (lane 4 t + q holds elements [32q, 32q + 32) of tile t), as a
// register-blocked product: each lane computes 4 tiles x 8 outputs (tile group
// g = lane >> 4; outputs 4j .. 4j + 3 and 64 + 4j .. 64 + 4j + 3 for j = lane & 15),
// so that per input k a lane issues three 16-byte shared loads (4 inputs, 8 matrix
// entries) for 32 fma.  The inputs reach that layout, and the results return to the
// quarter layout, through a per-warp shared buffer.  Shared memory of a CTA of W
// warps, 16-byte aligned, rot_smem_bytes(W): M as S[k][o] = M[o][k] (row k over the
// 128 outputs, pitch kRotPitch), then one buffer of kRotBufFloats per warp.
constexpr int kRotPitch = 132;          // 16-byte rows; transposing writes at most 4-way bank conflicts
constexpr int kRotBufFloats = 8 * 132;  // inputs k-major 8 k + t + 8 (k >> 5), or results 132 t + o
__host__ __device__ constexpr size_t rot_smem_bytes(int warps) {
    return ((size_t)128 * kRotPitch + (size_t)warps * kRotBufFloats) * sizeof(float);
}
constexpr size_t kRotSmemBytes = rot_smem_bytes(kWarpsPerCta);

// Shared form of M from the row-major fp32 Q in global memory (coalesced reads, by the
// whole CTA): M = Q when FORWARD, else M = Q^T.  The caller synchronises.
template <bool FORWARD>
__device__ __forceinline__ void load_rotation(float *S, const float *Q) {
    for (int idx = threadIdx.x; idx < 128 * 128; idx += blockDim.x) {
        const int a = idx >> 7, b = idx & 127;
        const float v = __ldg(Q + idx);
        if (FORWARD)
            S[b * kRotPitch + a] = v;   // M[a][b] = Q[a][b]: output a, input b
        else
            S[a * kRotPitch + b] = v;   // M[b][a] = Q[a][b]: output b, input a
    }
}

// v (16 float2 per lane: v[i] = elements 2i, 2i + 1 of the lane's quarter) <- M v for
// each of the warp's eight tiles.  Whole warp; S as load_rotation leaves it.
__device__ __forceinline__ void rotate_round(float2 (&v)[16], const float *S, int lane) {
    float *buf = const_cast<float *>(S) + 128 * kRotPitch + (threadIdx.x >> 5) * kRotBufFloats;
    const int t = lane >> 2, q = lane & 3;
    // inputs, k-major: the 32 lanes of one store hit 32 distinct banks
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const int k = 32 * q + 2 * i;
        buf[8 * k + t + 8 * q] = v[i].x;
        buf[8 * (k + 1) + t + 8 * q] = v[i].y;
    }
    __syncwarp();
    const int g = lane >> 4, j = lane & 15;
    float2 acc[4][4];   // [tile 4g + tt][outputs (4j, 4j+1), (4j+2, 4j+3), (64+4j, ..), (66+4j, ..)]
#pragma unroll
    for (int tt = 0; tt < 4; tt++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[tt][c] = make_float2(0.0f, 0.0f);
#pragma unroll 8
    for (int k = 0; k < 128; k++) {
        const float4 z = *reinterpret_cast<const float4 *>(buf + 8 * k + 8 * (k >> 5) + 4 * g);
        const float4 m0 = *reinterpret_cast<const float4 *>(S + k * kRotPitch + 4 * j);
        const float4 m1 = *reinterpret_cast<const float4 *>(S + k * kRotPitch + 64 + 4 * j);
        const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
        for (int tt = 0; tt < 4; tt++) {
            const float2 x2 = make_float2(zz[tt], zz[tt]);
            acc[tt][0] = f2_fma(make_float2(m0.x, m0.y), x2, acc[tt][0]);
            acc[tt][1] = f2_fma(make_float2(m0.z, m0.w), x2, acc[tt][1]);
            acc[tt][2] = f2_fma(make_float2(m1.x, m1.y), x2, acc[tt][2]);
            acc[tt][3] = f2_fma(make_float2(m1.z, m1.w), x2, acc[tt][3]);
        }
    }
    __syncwarp();
    // results, tile-major
#pragma unroll
    for (int tt = 0; tt < 4; tt++) {
        float *row = buf + kRotPitch * (4 * g + tt);
        *reinterpret_cast<float4 *>(row + 4 * j) = make_float4(acc[tt][0].x, acc[tt][0].y, acc[tt][1].x, acc[tt][1].y);
        *reinterpret_cast<float4 *>(row + 64 + 4 * j) =
            make_float4(acc[tt][2].x, acc[tt][2].y, acc[tt][3].x, acc[tt][3].y);
    }
    __syncwarp();
    const float *row = buf + kRotPitch * t + 32 * q;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float4 r = *reinterpret_cast<const float4 *>(row + 4 * i);
        v[2 * i] = make_float2(r.x, r.y);
        v[2 * i + 1] = make_float2(r.z, r.w);
    }
    __syncwarp();
}

// v (4 float2 per lane: elements 8 l, 8 l + 1, ..., 8 l + 7 of the half-warp's tile, l =
// lane & 15, the wide layout) <- M v for each half-warp's tile.  Each lane computes its own
// 8 outputs: per input k, two 16-byte loads of S[k][8 l ..] (the other half-warp reads the
// same words) and a 16-byte broadcast of 4 inputs from xs, the half-warp's 128-float copy
// of its tile (16-byte aligned, at xs + 128 * (lane >> 4)).  Whole warp.
__device__ __forceinline__ void rotate_sixteenth(float2 (&v)[4], const float *S, float *xs, int lane) {
    const int l16 = lane & 15;
    float *x = xs + 128 * (lane >> 4);
    reinterpret_cast<float4 *>(x)[2 * l16] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    reinterpret_cast<float4 *>(x)[2 * l16 + 1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
    __syncwarp();
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < 4; c++) acc[c] = make_float2(0.0f, 0.0f);
#pragma unroll 4
    for (int k4 = 0; k4 < 32; k4++) {
        const float4 x4 = reinterpret_cast<const float4 *>(x)[k4];
        const float xk[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const float *row = S + (4 * k4 + u) * kRotPitch + 8 * l16;
            const float4 m0 = *reinterpret_cast<const float4 *>(row);
            const float4 m1 = *reinterpret_cast<const float4 *>(row + 4);
            const float2 x2 = make_float2(xk[u], xk[u]);
            acc[0] = f2_fma(make_float2(m0.x, m0.y), x2, acc[0]);
            acc[1] = f2_fma(make_float2(m0.z, m0.w), x2, acc[1]);
            acc[2] = f2_fma(make_float2(m1.x, m1.y), x2, acc[2]);
            acc[3] = f2_fma(make_float2(m1.z, m1.w), x2, acc[3]);
        }
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; c++) v[c] = acc[c];
}

// ------------------------------------------------------------------ lattices
// Rounding without the conversion pipe: for |x| < 2^22, x + 1.5*2^23 lands in
// [2^23, 2^24) where the fp32 spacing is 1, so the add rounds x to the nearest
// integer with ties to even (1.5*2^23 is even), exactly like rint; subtracting
// the constant gives rint(x) as a float, and the integer is the bit pattern minus
// that of the constant.  Larger |x| are outside the supported range: they give
// large codes, which the range check (symbols >= 2^22) flags.
constexpr float kRoundMagic = 12582912.0f;
constexpr int32_t kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int32_t rint_int(float x) {
    return __float_as_int(__fadd_rn(x, kRoundMagic)) - kRoundMagicBits;
}

// D_n nearest point (Conway & Sloane) on one candidate: round every coordinate
// to nearest-even; if the integer sum is odd, move the coordinate farthest from
// its integer (first index on ties) one step toward its input.  Branch-free:
// the argmax is a compare/select chain and the step is a predicated add.
// In: t[i] = y[i] + kRoundMagic (rounded), f[i] = t[i] - kRoundMagic, r[i] = y[i] - f[i].
// Out: f[] with the fix applied.
template <int N>
__device__ __forceinline__ void dn_fix(const float (&r)[N], uint32_t par, float (&f)[N]) {
    float rb = r[0];
    int j = 0;
#pragma unroll
    for (int i = 1; i < N; i++) {
        const bool gt = fabsf(r[i]) > fabsf(rb);
        rb = gt ? r[i] : rb;
        j = gt ? i : j;
    }
    const float d = (par & 1u) ? ((rb >= 0.0f) ? 1.0f : -1.0f) : 0.0f;
#pragma unroll
    for (int i = 0; i < N; i++) f[i] = __fadd_rn(f[i], (i == j) ? d : 0.0f);
}

// sqrt(3)-related constants of the A2 embedding, rounded to fp32.
#define HQ_INV_SQRT3 0.57735026918962576451f
#define HQ_SQRT3_2 0.86602540378443864676f
#define HQ_SQRT3 1.73205080756887729353f

__device__ __forceinline__ uint32_t zigzag(int32_t m);

template <int LAT> struct Lattice;

// Z: plain rounding; symbol = code.
template <> struct Lattice<HQ_Z> {
    static constexpr int N = 1;
    __device__ static __forceinline__ void nearest(const float (&v)[1], int32_t (&q)[1]) { q[0] = rint_int(v[0]); }
    __device__ static __forceinline__ uint32_t symbols(const float (&v)[1], uint32_t (&z)[1], uint32_t &key) {
        z[0] = zigzag(rint_int(v[0]));
        key = max(key, z[0]);
        return 0;
    }
    __device__ static __forceinline__ void point(const int32_t (&q)[1], float (&p)[1]) { p[0] = (float)q[0]; }
    __device__ static __forceinline__ float box(int) { return 1.0f; }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[1], uint32_t, int32_t (&q)[1]) { q[0] = m[0]; }
};

// D4 = {q in Z^4 : sum even}; q3's parity is implied by q0 + q1 + q2.
template <> struct Lattice<HQ_D4> {
    static constexpr int N = 4;
    __device__ static __forceinline__ void nearest(const float (&v)[4], int32_t (&q)[4]) {
        float f[4], r[4];
        uint32_t par = 0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float t = __fadd_rn(v[i], kRoundMagic);
            f[i] = __fsub_rn(t, kRoundMagic);
            r[i] = __fsub_rn(v[i], f[i]);
            par ^= __float_as_uint(t);
        }
        dn_fix<4>(r, par, f);
#pragma unroll
        for (int i = 0; i < 4; i++) q[i] = rint_int(f[i]);
    }
    __device__ static __forceinline__ uint32_t symbols(const float (&v)[4], uint32_t (&z)[4], uint32_t &key) {
        int32_t q[4];
        nearest(v, q);
        z[0] = zigzag(q[0]);
        z[1] = zigzag(q[1]);
        z[2] = zigzag(q[2]);
        z[3] = zigzag((q[3] - ((q[0] + q[1] + q[2]) & 1)) >> 1);
        key = max(max(key, max(z[0], z[1])), max(z[2], zigzag(q[3])));
        return 0;
    }
    __device__ static __forceinline__ void point(const int32_t (&q)[4], float (&p)[4]) {
#pragma unroll
        for (int i = 0; i < 4; i++) p[i] = (float)q[i];
    }
    __device__ static __forceinline__ float box(int) { return 2.0f; }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[4], uint32_t, int32_t (&q)[4]) {
        q[0] = m[0];
        q[1] = m[1];
        q[2] = m[2];
        q[3] = 2 * m[3] + ((m[0] + m[1] + m[2]) & 1);
    }
};

// A2 at unit minimum distance: code (a, b), a = b mod 2, point (a/2, b sqrt(3)/2);
// union of Z x sqrt(3)Z (even codes) and its translate by (1/2, sqrt(3)/2) (odd
// codes); nearest point of each rectangular coset, the nearer wins (even on ties).
template <> struct Lattice<HQ_A2> {
    static constexpr int N = 2;
    __device__ static __forceinline__ void point(const int32_t (&q)[2], float (&p)[2]) {
        p[0] = __fmul_rn((float)q[0], 0.5f);
        p[1] = __fmul_rn((float)q[1], HQ_SQRT3_2);
    }
    __device__ static __forceinline__ void nearest(const float (&u)[2], int32_t (&q)[2]) {
        const float t1 = __fmul_rn(u[1], HQ_INV_SQRT3);
        const int32_t c0a = 2 * rint_int(u[0]), c0b = 2 * rint_int(t1);
        const int32_t c1a = 2 * rint_int(__fsub_rn(u[0], 0.5f)) + 1, c1b = 2 * rint_int(__fsub_rn(t1, 0.5f)) + 1;
        float r, d0 = 0.0f, d1 = 0.0f;
        r = __fsub_rn(u[0], __fmul_rn((float)c0a, 0.5f)); d0 = __fmaf_rn(r, r, d0);
        r = __fsub_rn(u[1], __fmul_rn((float)c0b, HQ_SQRT3_2)); d0 = __fmaf_rn(r, r, d0);
        r = __fsub_rn(u[0], __fmul_rn((float)c1a, 0.5f)); d1 = __fmaf_rn(r, r, d1);
        r = __fsub_rn(u[1], __fmul_rn((float)c1b, HQ_SQRT3_2)); d1 = __fmaf_rn(r, r, d1);
        const bool odd = d1 < d0;
        q[0] = odd ? c1a : c0a;
        q[1] = odd ? c1b : c0b;
    }
    __device__ static __forceinline__ uint32_t symbols(const float (&u)[2], uint32_t (&z)[2], uint32_t &key) {
        int32_t q[2];
        nearest(u, q);
        z[0] = zigzag(q[0]);
        z[1] = zigzag((q[1] - (q[0] & 1)) >> 1);
        key = max(key, max(z[0], zigzag(q[1])));
        return 0;
    }
    __device__ static __forceinline__ float box(int i) { return (i & 1) ? HQ_SQRT3 : 1.0f; }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[2], uint32_t, int32_t (&q)[2]) {
        q[0] = m[0];
        q[1] = 2 * m[1] + (m[0] & 1);
    }
};

// E8 as 2E8 = 2D8 u (2D8 + 1) in Z^8: candidate A = 2 D8(v/2), candidate
// B = 2 D8((v - 1)/2) + 1, keep B only if strictly nearer by the sequential
// fma distance in index order (the reading of the decoder).  The symbols come
// straight from the D8 integers m of the winner: coset bit c (0 for A, 1 for B),
// m_i = (q_i - c)/2, and m_7's parity (implied by m_0..m_6) is stripped.
//
// Exact decision, fast.  Both candidates' D8 points are found exactly as the
// reading defines them (two candidates side by side in packed fp32 operations).
// Only the distance comparison is estimated: with r = y - rint(y), a parity fix
// moves the coordinate of largest |r| to residual 1 - |r|, so candidate X's
// squared distance / 4 is S_X + p_X (1 - 2 max|r|) with S_X = sum r^2, in real
// arithmetic (for B up to the rounding of v - 1).  Over both candidates the
// estimates differ from the reading's fp32 sequential-fma distances / 4 by at most
// 19.01u (E_A + E_B) + u sum|v| + 10u (u = 2^-24; terms: the reading's rounded
// residuals and 8-step fma chain, 10.01u E each; this estimate's sum of squares (two
// 4-step fma chains over alternate coordinates and their sum) and two roundings, at
// most 9u E + u each; the rounding of v - 1 in candidate B, u (sum|v| + 8)).
// The margin below, 2^-18 (E_A + E_B + 4) + 2^-21 sum|v| = 64u (E_A + E_B) + 256u
// + 8u sum|v|, is at least 3.3 times that bound.  Outside the margin the estimate
// decides; inside it (near-ties, exact ties, huge inputs) the reading's own
// distances are rebuilt from the same rounded values (exact_dist).
template <> struct Lattice<HQ_E8> {
    static constexpr int N = 8;
    __device__ static __forceinline__ void point(const int32_t (&q)[8], float (&p)[8]) {
#pragma unroll
        for (int i = 0; i < 8; i++) p[i] = (float)q[i];
    }
    // Index of the largest |r_i| (first on ties) and r at that index.
    __device__ static __forceinline__ int argmax_abs(const float (&r)[8], float &rb) {
        rb = r[0];
        int j = 0;
#pragma unroll
        for (int i = 1; i < 8; i++) {
            const bool gt = fabsf(r[i]) > fabsf(rb);
            rb = gt ? r[i] : rb;
            j = gt ? i : j;
        }
        return j;
    }
    // The reading's sequential fma distance of one candidate, rebuilt from its rounded
    // values (t = y + 1.5 * 2^23), residuals r and parity: the fixed D8 point f, the
    // embedded point 2 f + c, then acc = fma(rho, rho, acc) in index order.
    __device__ static __forceinline__ float exact_dist(const float (&v)[8], const uint32_t (&t)[8],
                                                       const float (&r)[8], uint32_t par, float c) {
        float rb;
        const int j = argmax_abs(r, rb);
        const float d = (par & 1u) ? ((rb >= 0.0f) ? 1.0f : -1.0f) : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float f = __fadd_rn(__fsub_rn(__uint_as_float(t[i]), kRoundMagic), (i == j) ? d : 0.0f);
            const float rho = __fsub_rn(v[i], __fmaf_rn(f, 2.0f, c));
            acc = __fmaf_rn(rho, rho, acc);
        }
        return acc;
    }
    // D8 coordinates m of the nearest point (after the winner's parity fix); returns the coset bit.
    //
    // The two candidates' halved inputs are y_A = v / 2 and y_B = fl((v - 1) / 2), formed
    // here for two coordinates at a time as y_A = v * 0.5 and y_B = y_A - 0.5: halving is
    // exact and rounding commutes with it, so fl(y_A - 0.5) = fl(v - 1) / 2 bit for bit.
    __device__ static __forceinline__ uint32_t nearest_d8(const float (&v)[8], int32_t (&m)[8]) {
        const float2 M2 = make_float2(kRoundMagic, kRoundMagic), H2 = make_float2(0.5f, 0.5f);
        uint32_t ta[8], tb[8];
        float ra[8], rb[8];
        float2 SA = make_float2(0.0f, 0.0f), SB = make_float2(0.0f, 0.0f);
        float ma = 0.0f, mb = 0.0f, sv = 0.0f;
        uint32_t pa = 0, pb = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 ya = f2_mul(make_float2(v[2 * j], v[2 * j + 1]), H2);
            const float2 yb = f2_sub(ya, H2);
            const float2 tA = f2_add(ya, M2), tB = f2_add(yb, M2);
            const float2 rA = f2_sub(ya, f2_sub(tA, M2)), rB = f2_sub(yb, f2_sub(tB, M2));
            ta[2 * j] = __float_as_uint(tA.x);
            ta[2 * j + 1] = __float_as_uint(tA.y);
            tb[2 * j] = __float_as_uint(tB.x);
            tb[2 * j + 1] = __float_as_uint(tB.y);
            ra[2 * j] = rA.x;
            ra[2 * j + 1] = rA.y;
            rb[2 * j] = rB.x;
            rb[2 * j + 1] = rB.y;
            pa ^= ta[2 * j] ^ ta[2 * j + 1];
            pb ^= tb[2 * j] ^ tb[2 * j + 1];
            SA = f2_fma(rA, rA, SA);
            SB = f2_fma(rB, rB, SB);
            ma = fmaxf(ma, fmaxf(fabsf(rA.x), fabsf(rA.y)));
            mb = fmaxf(mb, fmaxf(fabsf(rB.x), fabsf(rB.y)));
            sv = __fadd_rn(__fadd_rn(sv, fabsf(v[2 * j])), fabsf(v[2 * j + 1]));
        }
        const float adja = (pa & 1u) ? __fmaf_rn(-2.0f, ma, 1.0f) : 0.0f;
        const float adjb = (pb & 1u) ? __fmaf_rn(-2.0f, mb, 1.0f) : 0.0f;
        const float2 E = make_float2(__fadd_rn(__fadd_rn(SA.x, SA.y), adja), __fadd_rn(__fadd_rn(SB.x, SB.y), adjb));
        const float diff = __fsub_rn(E.x, E.y);
        const float margin =
            __fmaf_rn(0x1p-21f, sv, __fmul_rn(0x1p-18f, __fadd_rn(__fadd_rn(E.x, E.y), 4.0f)));
        bool odd = diff > 0.0f;
        if (fabsf(diff) <= margin) odd = exact_dist(v, tb, rb, pb, 1.0f) < exact_dist(v, ta, ra, pa, 0.0f);
        // the winner's parity fix: coordinate of largest |r| (first on ties) one step toward y
        float rsel[8];
#pragma unroll
        for (int i = 0; i < 8; i++) rsel[i] = odd ? rb[i] : ra[i];
        float rw;
        const int j = argmax_abs(rsel, rw);
        const uint32_t pw = odd ? pb : pa;
        const int32_t d = (pw & 1u) ? ((rw >= 0.0f) ? 1 : -1) : 0;
#pragma unroll
        for (int i = 0; i < 8; i++)
            m[i] = (int32_t)((odd ? tb[i] : ta[i]) - (uint32_t)kRoundMagicBits) + ((i == j) ? d : 0);
        return odd ? 1u : 0u;
    }
    __device__ static __forceinline__ void nearest(const float (&v)[8], int32_t (&q)[8]) {
        int32_t m[8];
        const int32_t c = (int32_t)nearest_d8(v, m);
#pragma unroll
        for (int i = 0; i < 8; i++) q[i] = 2 * m[i] + c;
    }
    __device__ static __forceinline__ uint32_t symbols(const float (&v)[8], uint32_t (&z)[8], uint32_t &key) {
        int32_t m[8];
        const uint32_t c = nearest_d8(v, m);
        const int32_t s = m[0] + m[1] + m[2] + m[3] + m[4] + m[5] + m[6];
        const uint32_t z7 = zigzag(m[7]);   // before the strip: the code q_7 = 2 m_7 + c
        m[7] = (m[7] - (s & 1)) >> 1;
#pragma unroll
        for (int i = 0; i < 8; i++) z[i] = zigzag(m[i]);
        // |2 m + c| is z + ((z ^ c) & 1) with z = zigzag(m): nondecreasing in z for a fixed c,
        // so the block's largest |code| comes from its largest zigzag value
        const uint32_t zm = max(max(max(z[0], z[1]), max(z[2], z[3])), max(max(z[4], z[5]), max(z[6], z7)));
        key = max(key, zm + ((zm ^ c) & 1u));
        return c;
    }
    __device__ static __forceinline__ float box(int) { return 4.0f; }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[8], uint32_t c, int32_t (&q)[8]) {
        int32_t s = 0;
#pragma unroll
        for (int i = 0; i < 7; i++) s += m[i];
#pragma unroll
        for (int i = 0; i < 7; i++) q[i] = 2 * m[i] + (int32_t)c;
        q[7] = 2 * (2 * m[7] + (s & 1)) + (int32_t)c;
    }
};

__device__ __forceinline__ uint32_t zigzag(int32_t m) { return ((uint32_t)m << 1) ^ (uint32_t)(m >> 31); }
__device__ __forceinline__ int32_t unzigzag(uint32_t z) { return (int32_t)(z >> 1) ^ -(int32_t)(z & 1u); }

// a * b + c in one integer multiply-add (b a runtime power of two: a Rice quotient
// shifted up by k without a shift instruction).
__device__ __forceinline__ uint32_t imad(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// E8 codes of a block straight from its 8 symbols and coset bit c: twice the zigzag
// inverse is 2m = z ^ -(z & 1) (bit 0 clear), so q_i = 2 m_i + c = (z_i ^ s_i) | c;
// the stripped parity of m_7 is bit 1 of q_0 ^ ... ^ q_6 (= the parity of sum m_i),
// and q_7 = 2 (2 m_7' + p) + c.  Equal to Lattice<E8>::reinsert of the unzigzagged m.
__device__ __forceinline__ void e8_codes_from_symbols(const uint32_t (&z)[8], uint32_t c, int32_t (&q)[8]) {
    uint32_t x = 0;
#pragma unroll
    for (int i = 0; i < 7; i++) {
        const uint32_t t = (z[i] ^ (0u - (z[i] & 1u))) | c;
        q[i] = (int32_t)t;
        x ^= t;
    }
    const uint32_t t7 = z[7] ^ (0u - (z[7] & 1u));
    q[7] = (int32_t)((t7 << 1) | (x & 2u) | c);
}

// ------------------------------------------------------------------ decoded points
// fp32 value of an integer code q with -2^22 <= q < 2^22, without the conversion pipe:
// 1.5 * 2^23 + q has spacing 1 there, so its bit pattern is that of the constant plus q
// and subtracting the constant is exact.
__device__ __forceinline__ float small_int_float(int32_t q) {
    return __fsub_rn(__int_as_float(q + kRoundMagicBits), kRoundMagic);
}
// The lattice point of decoded codes (Lattice<LAT>::point), for codes rebuilt from
// symbols below 2^22 (the encoder flags larger ones): every coordinate except E8's last,
// whose code (4 m_7' + 2 p + c) may reach 2^23, is in small_int_float's range.
template <int LAT>
__device__ __forceinline__ void decoded_point(const int32_t (&q)[Lattice<LAT>::N], float (&p)[Lattice<LAT>::N]) {
    if constexpr (LAT == HQ_A2) {
        p[0] = __fmul_rn(small_int_float(q[0]), 0.5f);
        p[1] = __fmul_rn(small_int_float(q[1]), HQ_SQRT3_2);
    } else {
        constexpr int N = Lattice<LAT>::N;
#pragma unroll
        for (int i = 0; i < N; i++) p[i] = (LAT == HQ_E8 && i == N - 1) ? (float)q[i] : small_int_float(q[i]);
    }
}

// ------------------------------------------------------------------ integer range of the codes
// The pages store the embedding's integers in 8 bits, with alpha chosen so that they fit
// (explainer pages, "Methodology" 2, the integer implementation); the encoders report the
// largest |code coordinate| and the number of coordinates outside [-128, 127].  symbols()
// keeps a per-lattice key of the largest |code|: E8 the value itself; Z, A2, D4 the zigzag
// value of the code coordinate, from which |q| = (key + 1) >> 1, and a coordinate lies
// outside int8 exactly when its zigzag value is 256 or more.
template <int LAT>
__device__ __forceinline__ uint32_t code_abs_of_key(uint32_t key) {
    return LAT == HQ_E8 ? key : (key >> 1) + (key & 1u);
}
// A key at or above this may hide a coordinate outside int8 (E8: |q| = 128 is fine for q = -128).
template <int LAT>
__device__ __forceinline__ uint32_t key_int8_limit() {
    return LAT == HQ_E8 ? 128u : 256u;
}

// Code coordinates outside [-128, 127] among S symbols (S / N whole lattice blocks, E8 coset
// bits in cbits, bit b for block b), rebuilt from the symbols.  The rare path: taken only when
// a key reached key_int8_limit.
template <int LAT, int S>
__device__ __noinline__ uint32_t int8_overflow(const uint32_t (&z)[S], uint32_t cbits) {
    constexpr int N = Lattice<LAT>::N;
    uint32_t n = 0;
#pragma unroll
    for (int b = 0; b < S / N; b++) {
        int32_t q[N];
        if constexpr (LAT == HQ_E8) {
            uint32_t zb[8];
#pragma unroll
            for (int i = 0; i < 8; i++) zb[i] = z[8 * b + i];
            e8_codes_from_symbols(zb, (cbits >> b) & 1u, q);
        } else {
            int32_t m[N];
#pragma unroll
            for (int i = 0; i < N; i++) m[i] = unzigzag(z[N * b + i]);
            Lattice<LAT>::reinsert(m, 0u, q);
        }
#pragma unroll
        for (int i = 0; i < N; i++) n += ((uint32_t)(q[i] + 128) > 255u) ? 1u : 0u;
    }
    return n;
}

// ------------------------------------------------------------------ dither
// Section 4 subtractive dither: uniform r in [0,1) from 24 bits of the
// generator output for pair e >> 1 (bits 40..63 for even e, 8..31 for odd e);
// w = box * r is uniform on a fundamental box of a sublattice of the embedding,
// and d = w - point(Q(w)) is uniform on the Voronoi cell.  e0 is even (tiles
// start at multiples of 128), so a block of N >= 2 coordinates uses N/2 hashes.
template <int LAT>
__device__ __forceinline__ void dither_block(uint64_t seed, uint64_t e0, float (&d)[Lattice<LAT>::N]) {
    constexpr int N = Lattice<LAT>::N;
    float w[N], p[N];
    int32_t q[N];
    const uint64_t sd = seed ^ kDitherSalt;
#pragma unroll
    for (int i = 0; i < N; i += 2) {
        uint64_t e = e0 + (uint64_t)i;
        uint64_t h = splitmix64(sd, e >> 1);
        float r0 = __fmul_rn((float)(uint32_t)(h >> 40), 0x1p-24f);
        w[i] = __fmul_rn(Lattice<LAT>::box(i), r0);
        if (i + 1 < N) {
            float r1 = __fmul_rn((float)((uint32_t)h >> 8), 0x1p-24f);
            w[i + 1] = __fmul_rn(Lattice<LAT>::box(i + 1), r1);
        }
    }
    Lattice<LAT>::nearest(w, q);
    Lattice<LAT>::point(q, p);
#pragma unroll
    for (int i = 0; i < N; i++) d[i] = __fsub_rn(w[i], p[i]);
}

// Z has one coordinate per block, so odd counters occur: generic per-element form.
template <>
__device__ __forceinline__ void dither_block<HQ_Z>(uint64_t seed, uint64_t e, float (&d)[1]) {
    uint64_t h = splitmix64(seed ^ kDitherSalt, e >> 1);
    uint32_t r24 = (e & 1ull) ? ((uint32_t)h >> 8) : (uint32_t)(h >> 40);
    float w = __fmul_rn((float)r24, 0x1p-24f);
    d[0] = __fsub_rn(w, (float)rint_int(w));
}

// ------------------------------------------------------------------ Rice parameters
// The Rice parameter of symbol i of a lane's run (its position i mod N in the lattice
// block): bit-stripping halves the last symbol of an A2, D4 or E8 block, which may take
// its own parameter kl (kl = k gives the single-parameter code).  Z has no such symbol.
template <int N>
__device__ __forceinline__ int sym_k(int i, int k, int kl) {
    return (N > 1 && (i % N) == N - 1) ? kl : k;
}
// Remainder bits of one 128-element tile, and of a group of 8 symbols.
template <int N>
__device__ __forceinline__ uint32_t tile_rem_bits(int k, int kl) {
    return N > 1 ? (uint32_t)(128 / N) * (uint32_t)((N - 1) * k + kl) : 128u * (uint32_t)k;
}
template <int N>
__device__ __forceinline__ uint32_t group_rem_bits(int k, int kl) {
    return N > 1 ? (uint32_t)(8 / N) * (uint32_t)((N - 1) * k + kl) : 8u * (uint32_t)k;
}

// ------------------------------------------------------------------ integer helpers
// q = a / b, r = a % b (b > 0) with one 32-bit division when both fit, which is the
// usual case for chunk and tile counts; the 64-bit division otherwise.
__device__ __forceinline__ void divmod_u64(unsigned long long a, unsigned long long b, unsigned long long &q,
                                           unsigned long long &r) {
    if (((a | b) >> 32) == 0) {
        const uint32_t qq = (uint32_t)a / (uint32_t)b;
        q = qq;
        r = (uint32_t)a - qq * (uint32_t)b;
    } else {
        q = a / b;
        r = a - q * b;
    }
}

// ------------------------------------------------------------------ memory helpers
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

}  // namespace hq
