/*
 * hqref.c -- plain, slow CPU oracle of the HyperQuant quantize / dequantize path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark load it.  It shares no header, table or helper with the CUDA
 * path: every constant below is written out here from its definition.
 *
 * Source of the method: "HyperQuant" explainer pages (gist.science, paper
 * 2606.23406, sections "Methodology": 1 per-tile RHT, 2 lattice quantization,
 * 3 bit-stripping and Rice coding, 4 KV bias correction) and the arXiv abstract
 * (items (i)-(iv)).  The pages give no constants, no bitstream and no code; the
 * readings taken where they are silent are marked [R1]..[R19] and listed in the
 * design notes of the repository.
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * fp32 arithmetic is IEEE round-to-nearest-even, no FMA contraction, no FTZ;
 * fmaf() is called only where a reading says so.
 *
 * Parity status of each function (what pins it) is given in its comment; the
 * tests under tests/ carry the pins.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "hqref.h"

/* ------------------------------------------------------------------------ */
/* Counter-based generator [R3]: the i-th output (i = 0, 1, ...) of Steele,
 * Lea and Flood's SplitMix64 started from state s.  Pinned by the published
 * reference vectors for state 1234567. */
uint64_t hqref_splitmix64(uint64_t s, uint64_t i)
{
    uint64_t z = s + (i + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Random sign diagonal D of the RHT [R3]: s_j = -1 iff the top bit of the
 * j-th generator output from state (seed xor "SIGN") is set.  j is the column
 * index of the element in its row (weights) or the head dimension (KV). */
int hqref_sign(uint64_t seed, uint64_t j)
{
    return (hqref_splitmix64(seed ^ 0x5349474Eull, j) >> 63) ? -1 : 1;
}

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32.  bf16 is the top half of an fp32 bit pattern. */
float hqref_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN -> quiet NaN). */
uint16_t hqref_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16, lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* Unnormalised Walsh-Hadamard transform of one 128-element tile [R2]:
 * Sylvester (natural) order, radix-2 stages h = 1, 2, 4, ..., 64; at each
 * stage every pair (i, i+h) with (i & h) == 0 becomes (a+b, a-b).  The
 * orthonormal H_n of the pages is this transform times 1/sqrt(128); that
 * factor is folded into the scale constants below. */
void hqref_fwht128(float *v)
{
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i++)
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

/* Scale alpha [R4]: forward factor c = alpha / sqrt(128), inverse factor
 * e = 1 / (alpha * sqrt(128)), each computed in double and rounded once. */
float hqref_scale_fwd(float alpha) { return (float)((double)alpha / sqrt(128.0)); }
float hqref_scale_inv(float alpha) { return (float)(1.0 / ((double)alpha * sqrt(128.0))); }

/* ------------------------------------------------------------------------ */
/* Lattice nearest-point decoders [R5]-[R8].  "round" is rintf() in the
 * default round-to-nearest-even mode. */

int hqref_lattice_dim(int lat)
{
    switch (lat) {
    case HQREF_Z:  return 1;
    case HQREF_A2: return 2;
    case HQREF_D4: return 4;
    case HQREF_E8: return 8;
    }
    return 0;
}

/* D_n = { x in Z^n : sum x even }.  Conway & Sloane's decoder: round every
 * coordinate; if the sum is odd, re-round the coordinate farthest from its
 * integer (first index on ties) the other way. */
static void dn_decode(const float *y, int n, int32_t *f)
{
    int32_t sum = 0;
    for (int i = 0; i < n; i++) {
        f[i] = (int32_t)rintf(y[i]);
        sum += f[i];
    }
    if (sum & 1) {
        int j = 0;
        float best = fabsf(y[0] - (float)f[0]);
        for (int i = 1; i < n; i++) {
            float d = fabsf(y[i] - (float)f[i]);
            if (d > best) {
                best = d;
                j = i;
            }
        }
        f[j] += (y[j] >= (float)f[j]) ? 1 : -1;
    }
}

/* Sequential squared distance, one fmaf per coordinate in index order [R6]. */
static float sqdist_int(const float *v, const int32_t *q, int n)
{
    float acc = 0.0f;
    for (int i = 0; i < n; i++) {
        float r = v[i] - (float)q[i];
        acc = fmaf(r, r, acc);
    }
    return acc;
}

/* E8 in the integer embedding 2E8 = 2D8 u (2D8 + 1), a subset of Z^8 [R6].
 * Candidate A = 2 D8(v/2) (all even), candidate B = 2 D8((v-1)/2) + 1 (all
 * odd); the one at smaller squared distance wins, A on ties. */
void hqref_decode_e8(const float *v, int32_t *q)
{
    float y[8];
    int32_t fa[8], fb[8], A[8], B[8];
    for (int i = 0; i < 8; i++) y[i] = v[i] * 0.5f;
    dn_decode(y, 8, fa);
    for (int i = 0; i < 8; i++) A[i] = 2 * fa[i];
    for (int i = 0; i < 8; i++) y[i] = (v[i] - 1.0f) * 0.5f;
    dn_decode(y, 8, fb);
    for (int i = 0; i < 8; i++) B[i] = 2 * fb[i] + 1;
    float dA = sqdist_int(v, A, 8);
    float dB = sqdist_int(v, B, 8);
    const int32_t *w = (dB < dA) ? B : A;
    for (int i = 0; i < 8; i++) q[i] = w[i];
}

/* D4 = { x in Z^4 : sum even } [R7]. */
void hqref_decode_d4(const float *v, int32_t *q) { dn_decode(v, 4, q); }

/* Z: plain rounding. */
void hqref_decode_z(const float *v, int32_t *q) { q[0] = (int32_t)rintf(v[0]); }

/* A2 at unit minimum distance, code (a, b) with a = b (mod 2) standing for the
 * point (a/2, b*sqrt(3)/2) [R8].  A2 is the union of the rectangular lattice
 * Z x sqrt(3)Z (a, b even) and its translate by (1/2, sqrt(3)/2) (a, b odd);
 * the nearest point of each is found coordinate-wise, the nearer one wins
 * (coset 0 on ties). */
#define HQREF_INV_SQRT3 ((float)(0.57735026918962576451))   /* 1/sqrt(3) */
#define HQREF_SQRT3_2   ((float)(0.86602540378443864676))   /* sqrt(3)/2 */
#define HQREF_SQRT3     ((float)(1.73205080756887729353))   /* sqrt(3)   */

void hqref_point(int lat, const int32_t *q, float *p)
{
    int n = hqref_lattice_dim(lat);
    if (lat == HQREF_A2) {
        p[0] = (float)q[0] * 0.5f;
        p[1] = (float)q[1] * HQREF_SQRT3_2;
        return;
    }
    for (int i = 0; i < n; i++) p[i] = (float)q[i];
}

void hqref_decode_a2(const float *u, int32_t *q)
{
    float t1 = u[1] * HQREF_INV_SQRT3;
    int32_t c0[2], c1[2];
    c0[0] = 2 * (int32_t)rintf(u[0]);
    c0[1] = 2 * (int32_t)rintf(t1);
    c1[0] = 2 * (int32_t)rintf(u[0] - 0.5f) + 1;
    c1[1] = 2 * (int32_t)rintf(t1 - 0.5f) + 1;
    float p0[2], p1[2];
    hqref_point(HQREF_A2, c0, p0);
    hqref_point(HQREF_A2, c1, p1);
    float r;
    float d0 = 0.0f, d1 = 0.0f;
    r = u[0] - p0[0]; d0 = fmaf(r, r, d0);
    r = u[1] - p0[1]; d0 = fmaf(r, r, d0);
    r = u[0] - p1[0]; d1 = fmaf(r, r, d1);
    r = u[1] - p1[1]; d1 = fmaf(r, r, d1);
    const int32_t *w = (d1 < d0) ? c1 : c0;
    q[0] = w[0];
    q[1] = w[1];
}

void hqref_decode(int lat, const float *v, int32_t *q)
{
    switch (lat) {
    case HQREF_Z:  hqref_decode_z(v, q); break;
    case HQREF_A2: hqref_decode_a2(v, q); break;
    case HQREF_D4: hqref_decode_d4(v, q); break;
    case HQREF_E8: hqref_decode_e8(v, q); break;
    }
}

/* hqref_decode on n consecutive blocks (a plain loop; used by tests that decode
 * many vectors at once). */
void hqref_decode_many(int lat, const float *v, int64_t n, int32_t *q)
{
    const int d = hqref_lattice_dim(lat);
    for (int64_t b = 0; b < n; b++) hqref_decode(lat, v + b * d, q + b * d);
}

/* Membership predicate of the integer embeddings (used by tests). */
int hqref_is_member(int lat, const int32_t *q)
{
    switch (lat) {
    case HQREF_Z: return 1;
    case HQREF_A2: return ((q[0] - q[1]) & 1) == 0;
    case HQREF_D4: return ((q[0] + q[1] + q[2] + q[3]) & 1) == 0;
    case HQREF_E8: {
        int32_t c = q[0] & 1, s = 0;
        for (int i = 0; i < 8; i++) {
            if ((q[i] & 1) != c) return 0;
            s += (q[i] - c) / 2;
        }
        return (s & 1) == 0;
    }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Subtractive dither [R13].  For element counter e the uniform r in [0,1) is
 * 24 bits of the generator output for pair p = e >> 1 from state
 * (seed xor "DITH"): bits 40..63 for even e, bits 8..31 for odd e.  The
 * box B = [0, b_0) x ... is a fundamental region of a sublattice of the
 * embedding (E8: 4Z^8, D4: 2Z^4, Z: Z, A2: Z x sqrt(3)Z), so w = b * r is
 * uniform on it and d = w - point(Q(w)) is uniform on the Voronoi cell. */
float hqref_dither_uniform(uint64_t seed, uint64_t e)
{
    uint64_t h = hqref_splitmix64(seed ^ 0x44495448ull, e >> 1);
    uint32_t r24 = (e & 1u) ? ((uint32_t)h >> 8) : (uint32_t)(h >> 40);
    return (float)r24 * 0x1p-24f;
}

static float box_side(int lat, int i)
{
    switch (lat) {
    case HQREF_E8: return 4.0f;
    case HQREF_D4: return 2.0f;
    case HQREF_A2: return (i & 1) ? HQREF_SQRT3 : 1.0f;
    default:       return 1.0f;
    }
}

/* d for the lattice block whose first coordinate has counter e0. */
void hqref_dither_block(int lat, uint64_t seed, uint64_t e0, float *d)
{
    int n = hqref_lattice_dim(lat);
    float w[8], p[8];
    int32_t q[8];
    for (int i = 0; i < n; i++)
        w[i] = box_side(lat, i) * hqref_dither_uniform(seed, e0 + (uint64_t)i);
    hqref_decode(lat, w, q);
    hqref_point(lat, q, p);
    for (int i = 0; i < n; i++) d[i] = w[i] - p[i];
}

/* ------------------------------------------------------------------------ */
/* Bit-stripping [R9]: membership constraints fix some bits of a code vector;
 * they are removed before coding.  E8: the coset bit c (all coordinates share
 * parity c) is kept raw; m_i = (q_i - c) / 2; sum m is even, so m_7's parity
 * is implied and m_7' = (m_7 - p) / 2 is coded.  D4: q_3's parity is implied.
 * A2: b's parity equals a's.  Z: nothing to strip.  Division by 2 is an
 * arithmetic shift of an even number, hence exact. */
void hqref_strip(int lat, const int32_t *q, int32_t *m, uint32_t *coset)
{
    *coset = 0;
    switch (lat) {
    case HQREF_Z: m[0] = q[0]; break;
    case HQREF_A2:
        m[0] = q[0];
        m[1] = (q[1] - (q[0] & 1)) >> 1;
        break;
    case HQREF_D4: {
        m[0] = q[0]; m[1] = q[1]; m[2] = q[2];
        int32_t p = (q[0] + q[1] + q[2]) & 1;
        m[3] = (q[3] - p) >> 1;
        break;
    }
    case HQREF_E8: {
        int32_t c = q[0] & 1, s = 0;
        for (int i = 0; i < 8; i++) m[i] = (q[i] - c) >> 1;
        for (int i = 0; i < 7; i++) s += m[i];
        int32_t p = s & 1;
        m[7] = (m[7] - p) >> 1;
        *coset = (uint32_t)c;
        break;
    }
    }
}

void hqref_reinsert(int lat, const int32_t *m, uint32_t coset, int32_t *q)
{
    switch (lat) {
    case HQREF_Z: q[0] = m[0]; break;
    case HQREF_A2:
        q[0] = m[0];
        q[1] = 2 * m[1] + (m[0] & 1);
        break;
    case HQREF_D4: {
        q[0] = m[0]; q[1] = m[1]; q[2] = m[2];
        q[3] = 2 * m[3] + ((m[0] + m[1] + m[2]) & 1);
        break;
    }
    case HQREF_E8: {
        int32_t c = (int32_t)coset, s = 0, mm[8];
        for (int i = 0; i < 7; i++) { mm[i] = m[i]; s += m[i]; }
        mm[7] = 2 * m[7] + (s & 1);
        for (int i = 0; i < 8; i++) q[i] = 2 * mm[i] + c;
        break;
    }
    }
}

/* Zigzag map of signed symbols to non-negative integers [R10]. */
uint32_t hqref_zigzag(int32_t m) { return m >= 0 ? 2u * (uint32_t)m : 2u * (uint32_t)(-(int64_t)m) - 1u; }
int32_t hqref_unzigzag(uint32_t z) { return (z & 1u) ? (int32_t)(-(int64_t)(z / 2u) - 1) : (int32_t)(z / 2u); }

/* ------------------------------------------------------------------------ */
/* Bit I/O, LSB-first inside little-endian 32-bit words, one bit at a time. */
static void put_bit(uint32_t *w, uint64_t pos, uint32_t bit)
{
    if (bit) w[pos >> 5] |= 1u << (pos & 31);
}
static uint32_t get_bit(const uint32_t *w, uint64_t pos) { return (w[pos >> 5] >> (pos & 31)) & 1u; }

/* Classic concatenated Rice code [R10], used by the tests to show that the
 * plane layout carries exactly the same codeword bits: for each symbol z,
 * floor(z / 2^k) zeros, a one, then the k low bits of z (LSB first). */
uint64_t hqref_rice_concat(const uint32_t *z, int64_t n, int k, uint32_t *out, uint64_t cap_words)
{
    uint64_t pos = 0;
    for (int64_t i = 0; i < n; i++) {
        uint64_t q = z[i] >> k;
        uint64_t need = pos + q + 1 + (uint64_t)k;
        if (out && need <= 32ull * cap_words) {
            pos += q;
            put_bit(out, pos++, 1);
            for (int b = 0; b < k; b++) put_bit(out, pos++, (z[i] >> b) & 1u);
        } else {
            pos = need;
        }
    }
    return pos;
}

int hqref_rice_concat_decode(const uint32_t *in, uint64_t nbits, int64_t n, int k, uint32_t *z)
{
    uint64_t pos = 0;
    for (int64_t i = 0; i < n; i++) {
        uint64_t q = 0;
        while (pos < nbits && !get_bit(in, pos)) { q++; pos++; }
        if (pos >= nbits) return -1;
        pos++;
        uint32_t r = 0;
        for (int b = 0; b < k; b++) {
            if (pos >= nbits) return -1;
            r |= get_bit(in, pos++) << b;
        }
        z[i] = (uint32_t)(q << k) | r;
    }
    return 0;
}

/* Rice parameter of the symbol at position i of its lattice block [R19]: the
 * last symbol of an A2, D4 or E8 block (b', q3', m7': the one whose implied
 * bit R9 strips) takes max(k - dk_last, 0); every other symbol takes k.  With
 * dk_last = 0 every symbol takes k. */
int hqref_symbol_k(int lat, int k, int dk_last, int i)
{
    int n = hqref_lattice_dim(lat);
    if (n > 1 && i == n - 1) return (k > dk_last) ? k - dk_last : 0;
    return k;
}

/* Concatenated Rice codes with a parameter per symbol (ks[i]); the same as
 * hqref_rice_concat when every ks[i] is k. */
uint64_t hqref_rice_concat_k(const uint32_t *z, int64_t n, const int32_t *ks, uint32_t *out, uint64_t cap_words)
{
    uint64_t pos = 0;
    for (int64_t i = 0; i < n; i++) {
        int k = ks[i];
        uint64_t q = z[i] >> k;
        uint64_t need = pos + q + 1 + (uint64_t)k;
        if (out && need <= 32ull * cap_words) {
            pos += q;
            put_bit(out, pos++, 1);
            for (int b = 0; b < k; b++) put_bit(out, pos++, (z[i] >> b) & 1u);
        } else {
            pos = need;
        }
    }
    return pos;
}

/* ------------------------------------------------------------------------ */
/* Chunk planes [R12].  A chunk holds the symbols of ntiles tiles in order
 * (symbol index = tile * 128 + coordinate).  Layout, each plane starting on a
 * word boundary: [coset plane: 1 bit per E8 block] [remainder plane: the k_i
 * low bits of each symbol i, in symbol order, at the running sum of the k_i
 * (i * k when every k_i = k)] [unary plane: per symbol, floor(z/2^k_i) zeros
 * then a one], k_i = hqref_symbol_k(lat, k, dk_last, i mod n).  Returns the
 * chunk's word count; writes only if it fits in cap. */
uint64_t hqref_encode_chunk(int lat, int k, const int32_t *q, int ntiles, uint32_t *out, uint64_t cap_words,
                            uint64_t *payload_bits, int dk_last)
{
    int n = hqref_lattice_dim(lat);
    int64_t nsym = (int64_t)ntiles * 128;
    int64_t nblk = nsym / n;
    uint32_t *z = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)nsym);
    uint32_t *cb = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)nblk);
    for (int64_t b = 0; b < nblk; b++) {
        int32_t m[8];
        hqref_strip(lat, q + b * n, m, &cb[b]);
        for (int i = 0; i < n; i++) z[b * n + i] = hqref_zigzag(m[i]);
    }
    uint64_t wc = (lat == HQREF_E8) ? (uint64_t)(nblk + 31) / 32 : 0;
    uint64_t rbits = 0, ubits = 0;
    for (int64_t i = 0; i < nsym; i++) {
        int ki = hqref_symbol_k(lat, k, dk_last, (int)(i % n));
        rbits += (uint64_t)ki;
        ubits += (uint64_t)(z[i] >> ki) + 1;
    }
    uint64_t wr = (rbits + 31) / 32;
    uint64_t wu = (ubits + 31) / 32;
    uint64_t total = wc + wr + wu;
    if (payload_bits) *payload_bits = ubits + rbits + ((lat == HQREF_E8) ? (uint64_t)nblk : 0);
    if (out && total <= cap_words) {
        memset(out, 0, sizeof(uint32_t) * (size_t)total);
        if (lat == HQREF_E8)
            for (int64_t b = 0; b < nblk; b++) put_bit(out, (uint64_t)b, cb[b]);
        uint32_t *rem = out + wc;
        uint64_t rpos = 0;
        for (int64_t i = 0; i < nsym; i++) {
            int ki = hqref_symbol_k(lat, k, dk_last, (int)(i % n));
            for (int b = 0; b < ki; b++) put_bit(rem, rpos++, (z[i] >> b) & 1u);
        }
        uint32_t *un = out + wc + wr;
        uint64_t pos = 0;
        for (int64_t i = 0; i < nsym; i++) {
            pos += z[i] >> hqref_symbol_k(lat, k, dk_last, (int)(i % n));
            put_bit(un, pos++, 1);
        }
    }
    free(z);
    free(cb);
    return total;
}

/* Inverse of hqref_encode_chunk.  Returns 0, or -1 if the words do not hold
 * exactly nsym unary terminators inside the chunk. */
int hqref_decode_chunk(int lat, int k, const uint32_t *w, uint64_t nwords, int ntiles, int32_t *q, int dk_last)
{
    int n = hqref_lattice_dim(lat);
    int64_t nsym = (int64_t)ntiles * 128;
    int64_t nblk = nsym / n;
    uint64_t wc = (lat == HQREF_E8) ? (uint64_t)(nblk + 31) / 32 : 0;
    uint64_t rbits = 0;
    for (int i = 0; i < n; i++) rbits += (uint64_t)hqref_symbol_k(lat, k, dk_last, i);
    rbits *= (uint64_t)nblk;
    uint64_t wr = (rbits + 31) / 32;
    if (nwords < wc + wr) return -1;
    const uint32_t *rem = w + wc, *un = w + wc + wr;
    uint64_t ubits = 32 * (nwords - wc - wr);
    uint64_t pos = 0, rpos = 0;
    for (int64_t b = 0; b < nblk; b++) {
        int32_t m[8];
        for (int i = 0; i < n; i++) {
            int ki = hqref_symbol_k(lat, k, dk_last, i);
            uint64_t qq = 0;
            while (pos < ubits && !get_bit(un, pos)) { qq++; pos++; }
            if (pos >= ubits) return -1;
            pos++;
            uint32_t r = 0;
            for (int t = 0; t < ki; t++) r |= get_bit(rem, rpos++) << t;
            m[i] = hqref_unzigzag((uint32_t)(qq << ki) | r);
        }
        uint32_t c = (lat == HQREF_E8) ? get_bit(w, (uint64_t)b) : 0;
        hqref_reinsert(lat, m, c, q + b * n);
    }
    /* every remaining unary bit must be zero padding */
    for (; pos < ubits; pos++)
        if (get_bit(un, pos)) return -1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The lattice stage of a transformed, scaled tile v (128 fp32): per block of
 * n coordinates [+ d, R13], nearest point [R6]-[R8]. */
static void quantize_blocks(const float *v, int lat, uint64_t seed, int dither, uint64_t e0, int32_t *q)
{
    int n = hqref_lattice_dim(lat);
    for (int b = 0; b < 128; b += n) {
        float blk[8];
        for (int i = 0; i < n; i++) blk[i] = v[b + i];
        if (dither) {
            float d[8];
            hqref_dither_block(lat, seed, e0 + (uint64_t)b, d);
            for (int i = 0; i < n; i++) blk[i] = blk[i] + d[i];
        }
        hqref_decode(lat, blk, q + b);
    }
}

/* Its inverse up to the scale: v = lattice point [- d] per block [R14]. */
static void dequantize_blocks(const int32_t *q, int lat, uint64_t seed, int dither, uint64_t e0, float *v)
{
    int n = hqref_lattice_dim(lat);
    for (int b = 0; b < 128; b += n) {
        float p[8];
        hqref_point(lat, q + b, p);
        if (dither) {
            float d[8];
            hqref_dither_block(lat, seed, e0 + (uint64_t)b, d);
            for (int i = 0; i < n; i++) p[i] = p[i] - d[i];
        }
        for (int i = 0; i < n; i++) v[b + i] = p[i];
    }
}

/* One tile, forward [R1]-[R6], [R13]: x (128 bf16) -> codes.  sign_col0 is the
 * sign index of element 0 (element i uses sign index sign_col0 + i); e0 is the
 * dither counter of element 0 (counters are consecutive along the tile). */
void hqref_quantize_tile(const uint16_t *x, int lat, float alpha, uint64_t seed, uint64_t sign_col0, int dither,
                         uint64_t e0, int32_t *q)
{
    float v[128];
    for (int i = 0; i < 128; i++) {
        float xi = hqref_bf16_to_f32(x[i]);
        v[i] = (hqref_sign(seed, sign_col0 + (uint64_t)i) < 0) ? -xi : xi;
    }
    hqref_fwht128(v);
    float c = hqref_scale_fwd(alpha);
    for (int i = 0; i < 128; i++) v[i] = v[i] * c;
    quantize_blocks(v, lat, seed, dither, e0, q);
}

/* One tile, inverse [R14]: codes -> fp32 reconstruction (before bf16 rounding). */
void hqref_dequantize_tile(const int32_t *q, int lat, float alpha, uint64_t seed, uint64_t sign_col0, int dither,
                           uint64_t e0, float *out)
{
    float v[128];
    dequantize_blocks(q, lat, seed, dither, e0, v);
    float e = hqref_scale_inv(alpha);
    for (int i = 0; i < 128; i++) v[i] = v[i] * e;
    hqref_fwht128(v);
    for (int i = 0; i < 128; i++)
        out[i] = (hqref_sign(seed, sign_col0 + (uint64_t)i) < 0) ? -v[i] : v[i];
}

/* ------------------------------------------------------------------------ */
/* Dense rotation of the KV path [R17] (explainer pages, "Methodology" 4: each
 * layer's keys and values are rotated either by a full Haar-uniform matrix or
 * by the cheap sign diagonal).  Q is a 128 x 128 orthogonal fp32 matrix,
 * row-major, and takes the place of H_128 D / sqrt(128):
 *   forward  y_i = sum_j Q[i][j] x_j,  u = y * alpha;
 *   inverse  z = (point [- d]) * fp32(1 / alpha),  x_j = sum_i Q[i][j] z_i.
 * Each sum is one fmaf per term, in increasing index, from +0.  Pinned by the
 * basis-vector cases (a single nonzero term is exact: a column or a row of Q)
 * and by the round trip Q^T (Q x) = x within fp32 rounding. */
void hqref_rotate_fwd(const float *Q, const float *x, float *y)
{
    for (int i = 0; i < 128; i++) {
        float acc = 0.0f;
        for (int j = 0; j < 128; j++) acc = fmaf(Q[i * 128 + j], x[j], acc);
        y[i] = acc;
    }
}

void hqref_rotate_inv(const float *Q, const float *z, float *x)
{
    for (int j = 0; j < 128; j++) {
        float acc = 0.0f;
        for (int i = 0; i < 128; i++) acc = fmaf(Q[i * 128 + j], z[i], acc);
        x[j] = acc;
    }
}

float hqref_scale_inv_rot(float alpha) { return (float)(1.0 / (double)alpha); }

void hqref_quantize_tile_rot(const uint16_t *x, int lat, float alpha, const float *Q, uint64_t seed, int dither,
                             uint64_t e0, int32_t *q)
{
    float xf[128], v[128];
    for (int i = 0; i < 128; i++) xf[i] = hqref_bf16_to_f32(x[i]);
    hqref_rotate_fwd(Q, xf, v);
    for (int i = 0; i < 128; i++) v[i] = v[i] * alpha;
    quantize_blocks(v, lat, seed, dither, e0, q);
}

void hqref_dequantize_tile_rot(const int32_t *q, int lat, float alpha, const float *Q, uint64_t seed, int dither,
                               uint64_t e0, float *out)
{
    float v[128];
    dequantize_blocks(q, lat, seed, dither, e0, v);
    float e = hqref_scale_inv_rot(alpha);
    for (int i = 0; i < 128; i++) v[i] = v[i] * e;
    hqref_rotate_inv(Q, v, out);
}

/* Gaussian draw e of the rotation generator [R18]: h = splitmix64(seed ^ "ROTN",
 * e), u1 = (hi32(h) + 1/2) 2^-32 in (0, 1), u2 = lo32(h) 2^-32 in [0, 1),
 * g = sqrt(-2 ln u1) cos(2 pi u2) (the Box-Muller transform, cosine branch), in
 * double.  Pinned by a Kolmogorov-Smirnov test against the normal CDF. */
double hqref_rot_gaussian(uint64_t seed, uint64_t e)
{
    const double two_pi = 6.283185307179586476925;
    uint64_t h = hqref_splitmix64(seed ^ 0x524F544EULL, e);
    double u1 = ((double)(h >> 32) + 0.5) * 0x1p-32;
    double u2 = (double)(h & 0xFFFFFFFFULL) * 0x1p-32;
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* ------------------------------------------------------------------------ */
/* Tile enumeration.  Weights [R1], [R12]: tiles in row-major order over an
 * R x C matrix (C % 128 == 0), chunk c = tiles [32c, 32c+32).  KV [R15]: an
 * append of T tokens of H heads makes, per head, ceil(T/32) chunks of up to 32
 * tokens; chunk order is head-major.  The dither counter of element (token,
 * head, dim) is (token * H + head) * 128 + dim; of weight element (r, col) it
 * is r * C + col. */
typedef struct {
    int kv;
    const uint16_t *x;
    int64_t rows, cols, ld;              /* weights */
    int64_t H, T, ld_tok, ld_head, tok0; /* kv */
    const float *rot;                    /* kv: dense rotation [R17], or NULL for H_128 D */
} tiles_t;

static int64_t n_chunks_of(const tiles_t *t)
{
    if (t->kv) return t->H * ((t->T + 31) / 32);
    int64_t nt = t->rows * (t->cols / 128);
    return (nt + 31) / 32;
}

/* tile i (0..31) of chunk c: pointer, sign column, dither counter; returns 0
 * if the chunk has no tile i. */
static int tile_of(const tiles_t *t, int64_t c, int i, const uint16_t **p, uint64_t *scol, uint64_t *e0,
                   int64_t *row_or_tok, int64_t *col_or_head)
{
    if (t->kv) {
        int64_t cph = (t->T + 31) / 32;
        int64_t h = c / cph, tc = c % cph;
        int64_t tok = tc * 32 + i;
        if (tok >= t->T) return 0;
        if (p) *p = t->x + h * t->ld_head + tok * t->ld_tok;
        *scol = 0;
        *e0 = (uint64_t)(((t->tok0 + tok) * t->H + h) * 128);
        *row_or_tok = tok;
        *col_or_head = h;
        return 1;
    }
    int64_t tpr = t->cols / 128;
    int64_t ti = c * 32 + i;
    if (ti >= t->rows * tpr) return 0;
    int64_t r = ti / tpr, tc = ti % tpr;
    if (p) *p = t->x + r * t->ld + tc * 128;
    *scol = (uint64_t)(tc * 128);
    *e0 = (uint64_t)(r * t->cols + tc * 128);
    *row_or_tok = r;
    *col_or_head = tc;
    return 1;
}

static int64_t encode_all(const tiles_t *t, int lat, float alpha, int k, uint64_t seed, int dither,
                          int64_t chunk_lo, int64_t chunk_hi, uint32_t *stream, uint64_t base_word,
                          uint64_t cap_words, uint64_t *offsets, uint64_t *payload_bits, int dk_last)
{
    int32_t *q = (int32_t *)malloc(sizeof(int32_t) * 32 * 128);
    uint64_t pos = base_word, pay = 0;
    int over = 0;
    for (int64_t c = chunk_lo; c < chunk_hi; c++) {
        int nt = 0;
        for (int i = 0; i < 32; i++) {
            const uint16_t *p;
            uint64_t scol, e0;
            int64_t a, b;
            if (!tile_of(t, c, i, &p, &scol, &e0, &a, &b)) break;
            if (t->rot)
                hqref_quantize_tile_rot(p, lat, alpha, t->rot, seed, dither, e0, q + i * 128);
            else
                hqref_quantize_tile(p, lat, alpha, seed, scol, dither, e0, q + i * 128);
            nt++;
        }
        uint64_t pb = 0;
        uint64_t room = (pos < cap_words) ? cap_words - pos : 0;
        uint64_t nw = hqref_encode_chunk(lat, k, q, nt, stream ? stream + pos : NULL, stream ? room : 0, &pb, dk_last);
        if (nw > room) over = 1;
        if (offsets) offsets[c - chunk_lo] = pos;
        pos += nw;
        pay += pb;
    }
    if (offsets) offsets[chunk_hi - chunk_lo] = pos;
    if (payload_bits) *payload_bits = pay;
    free(q);
    return over ? -(int64_t)pos : (int64_t)pos;
}

static int decode_all(const tiles_t *t, int lat, float alpha, int k, uint64_t seed, int dither, int64_t chunk_lo,
                      int64_t chunk_hi, const uint32_t *stream, const uint64_t *offsets, int out_fp32, void *out,
                      int64_t out_ld, int64_t out_ld_head, int64_t len, int dk_last)
{
    int32_t *q = (int32_t *)malloc(sizeof(int32_t) * 32 * 128);
    int bad = 0;
    for (int64_t c = chunk_lo; c < chunk_hi; c++) {
        int nt = 0;
        int64_t rt[32], ch[32];
        uint64_t sc[32], ee[32];
        for (int i = 0; i < 32; i++) {
            if (!tile_of(t, c, i, NULL, &sc[i], &ee[i], &rt[i], &ch[i])) break;
            nt++;
        }
        uint64_t w0 = offsets[c - chunk_lo], w1 = offsets[c - chunk_lo + 1];
        if (w1 < w0 || hqref_decode_chunk(lat, k, stream + w0, w1 - w0, nt, q, dk_last) != 0) {
            bad = 1;
            continue;
        }
        for (int i = 0; i < nt; i++) {
            float f[128];
            if (t->rot)
                hqref_dequantize_tile_rot(q + i * 128, lat, alpha, t->rot, seed, dither, ee[i], f);
            else
                hqref_dequantize_tile(q + i * 128, lat, alpha, seed, sc[i], dither, ee[i], f);
            int64_t off;
            if (t->kv) {
                int64_t tok = t->tok0 + rt[i];
                if (tok >= len) continue;
                off = ch[i] * out_ld_head + tok * out_ld;
            } else {
                off = rt[i] * out_ld + ch[i] * 128;
            }
            if (out_fp32) {
                float *o = (float *)out + off;
                for (int j = 0; j < 128; j++) o[j] = f[j];
            } else {
                uint16_t *o = (uint16_t *)out + off;
                for (int j = 0; j < 128; j++) o[j] = hqref_f32_to_bf16(f[j]);
            }
        }
    }
    free(q);
    return bad ? -1 : 0;
}

/* [R11] The codes against 8-bit storage.  The pages store the lattice points'
 * integers in 8 bits and calibrate alpha so that they do not overflow
 * (explainer pages, "Methodology" 2, the integer implementation); the Rice
 * code is unbounded, so nothing is clamped and the range is only reported:
 * over the n code coordinates q (the embedding's integers, before
 * bit-stripping), the largest |q_i| is kept in *max_abs if it is larger, and
 * the number of q_i outside [-128, 127] is added to *overflow. */
void hqref_code_range(const int32_t *q, int64_t n, uint32_t *max_abs, uint64_t *overflow)
{
    for (int64_t i = 0; i < n; i++) {
        int64_t v = q[i];
        uint64_t a = (uint64_t)(v < 0 ? -v : v);
        if (a > *max_abs) *max_abs = (uint32_t)a;
        if (v < -128 || v > 127) *overflow += 1;
    }
}

/* The code range of every tile of chunks [chunk_lo, chunk_hi), from the same
 * per-tile quantization as encode_all. */
static void range_all(const tiles_t *t, int lat, float alpha, uint64_t seed, int dither, int64_t chunk_lo,
                      int64_t chunk_hi, uint32_t *max_abs, uint64_t *overflow)
{
    int32_t q[128];
    *max_abs = 0;
    *overflow = 0;
    for (int64_t c = chunk_lo; c < chunk_hi; c++) {
        for (int i = 0; i < 32; i++) {
            const uint16_t *p;
            uint64_t scol, e0;
            int64_t a, b;
            if (!tile_of(t, c, i, &p, &scol, &e0, &a, &b)) break;
            if (t->rot)
                hqref_quantize_tile_rot(p, lat, alpha, t->rot, seed, dither, e0, q);
            else
                hqref_quantize_tile(p, lat, alpha, seed, scol, dither, e0, q);
            hqref_code_range(q, 128, max_abs, overflow);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Whole-matrix API (weights). */
int64_t hqref_n_chunks(int64_t rows, int64_t cols)
{
    tiles_t t = {0};
    t.rows = rows;
    t.cols = cols;
    return n_chunks_of(&t);
}

int64_t hqref_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int lat, float alpha, int k,
                       uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi, uint32_t *stream,
                       uint64_t cap_words, uint64_t *offsets, uint64_t *payload_bits, int dk_last)
{
    tiles_t t = {0};
    t.x = x;
    t.rows = rows;
    t.cols = cols;
    t.ld = ld;
    return encode_all(&t, lat, alpha, k, seed, dither, chunk_lo, chunk_hi, stream, 0, cap_words, offsets,
                      payload_bits, dk_last);
}

int hqref_dequantize(const uint32_t *stream, const uint64_t *offsets, int64_t rows, int64_t cols, int lat,
                     float alpha, int k, uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi,
                     int out_fp32, void *out, int64_t ld, int dk_last)
{
    tiles_t t = {0};
    t.rows = rows;
    t.cols = cols;
    return decode_all(&t, lat, alpha, k, seed, dither, chunk_lo, chunk_hi, stream, offsets, out_fp32, out, ld, 0,
                      0, dk_last);
}

/* [R11] code range of a weight matrix's chunks [chunk_lo, chunk_hi). */
void hqref_quantize_range(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int lat, float alpha,
                          uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi, uint32_t *max_abs,
                          uint64_t *overflow)
{
    tiles_t t = {0};
    t.x = x;
    t.rows = rows;
    t.cols = cols;
    t.ld = ld;
    range_all(&t, lat, alpha, seed, dither, chunk_lo, chunk_hi, max_abs, overflow);
}

/* [R11] code range of one KV append (the tokens of hqref_kv_append's arguments). */
void hqref_kv_range(const uint16_t *kv, int64_t H, int64_t T, int64_t ld_tok, int64_t ld_head, int64_t tok0,
                    int lat, float alpha, uint64_t seed, int dither, const float *rot, uint32_t *max_abs,
                    uint64_t *overflow)
{
    tiles_t t = {0};
    t.kv = 1;
    t.x = kv;
    t.H = H;
    t.T = T;
    t.ld_tok = ld_tok;
    t.ld_head = ld_head;
    t.tok0 = tok0;
    t.rot = rot;
    range_all(&t, lat, alpha, seed, dither, 0, n_chunks_of(&t), max_abs, overflow);
}

/* KV append [R15]: the chunks of one append are written from base_word on;
 * offsets gets n_chunks + 1 entries (absolute word indices).  rot: the dense
 * rotation [R17], or NULL for H_128 D. */
int64_t hqref_kv_append(const uint16_t *kv, int64_t H, int64_t T, int64_t ld_tok, int64_t ld_head, int64_t tok0,
                        int lat, float alpha, int k, uint64_t seed, int dither, uint32_t *stream,
                        uint64_t base_word, uint64_t cap_words, uint64_t *offsets, uint64_t *payload_bits,
                        const float *rot, int dk_last)
{
    tiles_t t = {0};
    t.kv = 1;
    t.x = kv;
    t.H = H;
    t.T = T;
    t.ld_tok = ld_tok;
    t.ld_head = ld_head;
    t.tok0 = tok0;
    t.rot = rot;
    return encode_all(&t, lat, alpha, k, seed, dither, 0, n_chunks_of(&t), stream, base_word, cap_words, offsets,
                      payload_bits, dk_last);
}

/* Decode the chunks of one append into out[h * out_ld_head + tok * out_ld_tok + dim],
 * tokens at or beyond len skipped. */
int hqref_kv_read_append(const uint32_t *stream, const uint64_t *offsets, int64_t H, int64_t T, int64_t tok0,
                         int lat, float alpha, int k, uint64_t seed, int dither, int out_fp32, void *out,
                         int64_t out_ld_tok, int64_t out_ld_head, int64_t len, const float *rot, int dk_last)
{
    tiles_t t = {0};
    t.kv = 1;
    t.H = H;
    t.T = T;
    t.tok0 = tok0;
    t.rot = rot;
    return decode_all(&t, lat, alpha, k, seed, dither, 0, n_chunks_of(&t), stream, offsets, out_fp32, out,
                      out_ld_tok, out_ld_head, len, dk_last);
}
