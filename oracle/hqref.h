/*
 * hqref.h -- declarations of the plain CPU oracle (hqref.c).
 *
 * TEST INFRASTRUCTURE ONLY: the oracle's own header.  The product library has
 * its own public header and includes nothing from this directory.
 */
#ifndef HQREF_H
#define HQREF_H

#include <stdint.h>

enum { HQREF_Z = 0, HQREF_A2 = 1, HQREF_D4 = 2, HQREF_E8 = 3 };

uint64_t hqref_splitmix64(uint64_t s, uint64_t i);
int hqref_sign(uint64_t seed, uint64_t j);
float hqref_bf16_to_f32(uint16_t b);
uint16_t hqref_f32_to_bf16(float f);
void hqref_fwht128(float *v);
float hqref_scale_fwd(float alpha);
float hqref_scale_inv(float alpha);

int hqref_lattice_dim(int lat);
void hqref_decode_e8(const float *v, int32_t *q);
void hqref_decode_d4(const float *v, int32_t *q);
void hqref_decode_z(const float *v, int32_t *q);
void hqref_decode_a2(const float *u, int32_t *q);
void hqref_decode(int lat, const float *v, int32_t *q);
void hqref_decode_many(int lat, const float *v, int64_t n, int32_t *q);
void hqref_point(int lat, const int32_t *q, float *p);
int hqref_is_member(int lat, const int32_t *q);

float hqref_dither_uniform(uint64_t seed, uint64_t e);
void hqref_dither_block(int lat, uint64_t seed, uint64_t e0, float *d);

void hqref_strip(int lat, const int32_t *q, int32_t *m, uint32_t *coset);
void hqref_reinsert(int lat, const int32_t *m, uint32_t coset, int32_t *q);
uint32_t hqref_zigzag(int32_t m);
int32_t hqref_unzigzag(uint32_t z);

uint64_t hqref_rice_concat(const uint32_t *z, int64_t n, int k, uint32_t *out, uint64_t cap_words);
int hqref_rice_concat_decode(const uint32_t *in, uint64_t nbits, int64_t n, int k, uint32_t *z);
int hqref_symbol_k(int lat, int k, int dk_last, int i);
uint64_t hqref_rice_concat_k(const uint32_t *z, int64_t n, const int32_t *ks, uint32_t *out, uint64_t cap_words);
uint64_t hqref_encode_chunk(int lat, int k, const int32_t *q, int ntiles, uint32_t *out, uint64_t cap_words,
                            uint64_t *payload_bits, int dk_last);
int hqref_decode_chunk(int lat, int k, const uint32_t *w, uint64_t nwords, int ntiles, int32_t *q, int dk_last);

void hqref_quantize_tile(const uint16_t *x, int lat, float alpha, uint64_t seed, uint64_t sign_col0, int dither,
                         uint64_t e0, int32_t *q);
void hqref_dequantize_tile(const int32_t *q, int lat, float alpha, uint64_t seed, uint64_t sign_col0, int dither,
                           uint64_t e0, float *out);

void hqref_rotate_fwd(const float *Q, const float *x, float *y);
void hqref_rotate_inv(const float *Q, const float *z, float *x);
float hqref_scale_inv_rot(float alpha);
void hqref_quantize_tile_rot(const uint16_t *x, int lat, float alpha, const float *Q, uint64_t seed, int dither,
                             uint64_t e0, int32_t *q);
void hqref_dequantize_tile_rot(const int32_t *q, int lat, float alpha, const float *Q, uint64_t seed, int dither,
                               uint64_t e0, float *out);
double hqref_rot_gaussian(uint64_t seed, uint64_t e);

void hqref_code_range(const int32_t *q, int64_t n, uint32_t *max_abs, uint64_t *overflow);
void hqref_quantize_range(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int lat, float alpha,
                          uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi, uint32_t *max_abs,
                          uint64_t *overflow);
void hqref_kv_range(const uint16_t *kv, int64_t H, int64_t T, int64_t ld_tok, int64_t ld_head, int64_t tok0,
                    int lat, float alpha, uint64_t seed, int dither, const float *rot, uint32_t *max_abs,
                    uint64_t *overflow);
int64_t hqref_n_chunks(int64_t rows, int64_t cols);
int64_t hqref_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int lat, float alpha, int k,
                       uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi, uint32_t *stream,
                       uint64_t cap_words, uint64_t *offsets, uint64_t *payload_bits, int dk_last);
int hqref_dequantize(const uint32_t *stream, const uint64_t *offsets, int64_t rows, int64_t cols, int lat,
                     float alpha, int k, uint64_t seed, int dither, int64_t chunk_lo, int64_t chunk_hi,
                     int out_fp32, void *out, int64_t ld, int dk_last);
int64_t hqref_kv_append(const uint16_t *kv, int64_t H, int64_t T, int64_t ld_tok, int64_t ld_head, int64_t tok0,
                        int lat, float alpha, int k, uint64_t seed, int dither, uint32_t *stream,
                        uint64_t base_word, uint64_t cap_words, uint64_t *offsets, uint64_t *payload_bits,
                        const float *rot, int dk_last);
int hqref_kv_read_append(const uint32_t *stream, const uint64_t *offsets, int64_t H, int64_t T, int64_t tok0,
                         int lat, float alpha, int k, uint64_t seed, int dither, int out_fp32, void *out,
                         int64_t out_ld_tok, int64_t out_ld_head, int64_t len, const float *rot, int dk_last);

#endif
