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

// ------------------------------------------------------------------ FWHT-128
// Unnormalised Walsh-Hadamard transform in Sylvester order, radix-2 stages
// h = 1, 2, ..., 64, pair (i, i + h) -> (a + b, a - b).  The tile is held as
// 64 float2 (elements 2j, 2j+1): stage 1 works inside each pair; for h >= 2
// the butterflies of elements 2j and 2j+1 are independent and share a packed
// add and a packed subtract.  The 1/sqrt(128) of the orthonormal H_128 is
// folded into the scale factors.
__device__ __forceinline__ void fwht128(float2 (&v)[kTile / 2]) {
#pragma unroll
    for (int j = 0; j < kTile / 2; j++) {
        float a = v[j].x, b = v[j].y;
        v[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < kTile / 2; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < kTile / 2; j++) {
            if ((j & hp) == 0) {
                float2 a = v[j], b = v[j + hp];
                v[j] = f2_add(a, b);
                v[j + hp] = f2_sub(a, b);
            }
        }
    }
}

// ------------------------------------------------------------------ lattices
// D_n nearest point (Conway & Sloane): round every coordinate to nearest-even;
// if the integer sum is odd, move the coordinate farthest from its integer
// (first index on ties) one step toward its input.
template <int N>
__device__ __forceinline__ void dn_nearest(const float (&y)[N], int32_t (&f)[N]) {
    float r[N];
    int32_t par = 0;
#pragma unroll
    for (int i = 0; i < N; i++) {
        float fi = rintf(y[i]);
        f[i] = __float2int_rn(fi);
        r[i] = __fsub_rn(y[i], fi);
        par ^= f[i];
    }
    float best = fabsf(r[0]);
    int j = 0;
#pragma unroll
    for (int i = 1; i < N; i++) {
        float a = fabsf(r[i]);
        bool gt = a > best;
        best = gt ? a : best;
        j = gt ? i : j;
    }
    if (par & 1) {
#pragma unroll
        for (int i = 0; i < N; i++)
            if (i == j) f[i] += (r[i] >= 0.0f) ? 1 : -1;
    }
}

// sqrt(3)-related constants of the A2 embedding, rounded to fp32.
#define HQ_INV_SQRT3 0.57735026918962576451f
#define HQ_SQRT3_2 0.86602540378443864676f
#define HQ_SQRT3 1.73205080756887729353f

template <int LAT> struct Lattice;

// Z: plain rounding; symbol = code.
template <> struct Lattice<HQ_Z> {
    static constexpr int N = 1;
    __device__ static __forceinline__ void nearest(const float (&v)[1], int32_t (&q)[1]) {
        q[0] = __float2int_rn(v[0]);
    }
    __device__ static __forceinline__ void point(const int32_t (&q)[1], float (&p)[1]) { p[0] = (float)q[0]; }
    __device__ static __forceinline__ float box(int) { return 1.0f; }
    __device__ static __forceinline__ uint32_t strip(const int32_t (&q)[1], int32_t (&m)[1]) {
        m[0] = q[0];
        return 0;
    }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[1], uint32_t, int32_t (&q)[1]) { q[0] = m[0]; }
};

// D4 = {q in Z^4 : sum even}; q3's parity is implied by q0 + q1 + q2.
template <> struct Lattice<HQ_D4> {
    static constexpr int N = 4;
    __device__ static __forceinline__ void nearest(const float (&v)[4], int32_t (&q)[4]) { dn_nearest<4>(v, q); }
    __device__ static __forceinline__ void point(const int32_t (&q)[4], float (&p)[4]) {
#pragma unroll
        for (int i = 0; i < 4; i++) p[i] = (float)q[i];
    }
    __device__ static __forceinline__ float box(int) { return 2.0f; }
    __device__ static __forceinline__ uint32_t strip(const int32_t (&q)[4], int32_t (&m)[4]) {
        m[0] = q[0];
        m[1] = q[1];
        m[2] = q[2];
        m[3] = (q[3] - ((q[0] + q[1] + q[2]) & 1)) >> 1;
        return 0;
    }
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
        float t1 = __fmul_rn(u[1], HQ_INV_SQRT3);
        int32_t c0[2] = {2 * __float2int_rn(u[0]), 2 * __float2int_rn(t1)};
        int32_t c1[2] = {2 * __float2int_rn(__fsub_rn(u[0], 0.5f)) + 1, 2 * __float2int_rn(__fsub_rn(t1, 0.5f)) + 1};
        float p0[2], p1[2];
        point(c0, p0);
        point(c1, p1);
        float r, d0 = 0.0f, d1 = 0.0f;
        r = __fsub_rn(u[0], p0[0]); d0 = __fmaf_rn(r, r, d0);
        r = __fsub_rn(u[1], p0[1]); d0 = __fmaf_rn(r, r, d0);
        r = __fsub_rn(u[0], p1[0]); d1 = __fmaf_rn(r, r, d1);
        r = __fsub_rn(u[1], p1[1]); d1 = __fmaf_rn(r, r, d1);
        bool odd = d1 < d0;
        q[0] = odd ? c1[0] : c0[0];
        q[1] = odd ? c1[1] : c0[1];
    }
    __device__ static __forceinline__ float box(int i) { return (i & 1) ? HQ_SQRT3 : 1.0f; }
    __device__ static __forceinline__ uint32_t strip(const int32_t (&q)[2], int32_t (&m)[2]) {
        m[0] = q[0];
        m[1] = (q[1] - (q[0] & 1)) >> 1;
        return 0;
    }
    __device__ static __forceinline__ void reinsert(const int32_t (&m)[2], uint32_t, int32_t (&q)[2]) {
        q[0] = m[0];
        q[1] = 2 * m[1] + (m[0] & 1);
    }
};

// E8 as 2E8 = 2D8 u (2D8 + 1) in Z^8: candidate A = 2 D8(v/2), candidate
// B = 2 D8((v - 1)/2) + 1, keep B only if strictly nearer (sequential fma
// distance).  Stripping: coset bit c raw; m_i = (q_i - c) / 2; m_7's parity is
// implied by m_0..m_6, so m_7' = (m_7 - p) / 2 is coded.
template <> struct Lattice<HQ_E8> {
    static constexpr int N = 8;
    __device__ static __forceinline__ void point(const int32_t (&q)[8], float (&p)[8]) {
#pragma unroll
        for (int i = 0; i < 8; i++) p[i] = (float)q[i];
    }
    __device__ static __forceinline__ void nearest(const float (&v)[8], int32_t (&q)[8]) {
        float y[8];
        int32_t fa[8], fb[8];
#pragma unroll
        for (int i = 0; i < 8; i++) y[i] = __fmul_rn(v[i], 0.5f);
        dn_nearest<8>(y, fa);
#pragma unroll
        for (int i = 0; i < 8; i++) y[i] = __fmul_rn(__fsub_rn(v[i], 1.0f), 0.5f);
        dn_nearest<8>(y, fb);
        float dA = 0.0f, dB = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float r = __fsub_rn(v[i], (float)(2 * fa[i]));
            dA = __fmaf_rn(r, r, dA);
        }
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float r = __fsub_rn(v[i], (float)(2 * fb[i] + 1));
            dB = __fmaf_rn(r, r, dB);
        }
        bool odd = dB < dA;
#pragma unroll
        for (int i = 0; i < 8; i++) q[i] = odd ? 2 * fb[i] + 1 : 2 * fa[i];
    }
    __device__ static __forceinline__ float box(int) { return 4.0f; }
    __device__ static __forceinline__ uint32_t strip(const int32_t (&q)[8], int32_t (&m)[8]) {
        int32_t c = q[0] & 1, s = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) m[i] = (q[i] - c) >> 1;
#pragma unroll
        for (int i = 0; i < 7; i++) s += m[i];
        m[7] = (m[7] - (s & 1)) >> 1;
        return (uint32_t)c;
    }
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
    d[0] = __fsub_rn(w, (float)__float2int_rn(w));
}

// ------------------------------------------------------------------ memory helpers
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

}  // namespace hq
