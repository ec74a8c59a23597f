"""The oracle's pins have power: a plausible mistake planted in a copy of the
oracle (on the CPU) makes at least one pin fail.

Each case edits one line of a copy of hqref.c, compiles it with the same flags,
routes the oracle through it and runs the pins that should notice.
"""
import pytest

import oracle as O
import test_oracle_pins as P
import test_oracle_range as PG
import test_oracle_rice_k as PK
import test_oracle_rotation as PR

# (what the mistake is, text to find, replacement, pins expected to catch it)
MUTANTS = [
    ("butterfly difference reversed", "v[i + h] = a - b;", "v[i + h] = b - a;",
     [P.test_fwht_is_sylvester_hadamard_matrix]),
    ("butterfly partner index off by one stage", "v[i + h] = a - b;", "v[i + (h & 63)] = a - b;",
     [P.test_fwht_is_sylvester_hadamard_matrix]),
    ("odd coset shifted the wrong way", "y[i] = (v[i] - 1.0f) * 0.5f;", "y[i] = (v[i] + 1.0f) * 0.5f;",
     [lambda: P.test_decoder_is_nearest_point_by_brute_force(O.E8)]),
    ("parity fix rounds the wrong way", "f[j] += (y[j] >= (float)f[j]) ? 1 : -1;",
     "f[j] += (y[j] >= (float)f[j]) ? -1 : 1;",
     [lambda: P.test_decoder_is_nearest_point_by_brute_force(O.D4), P.test_dn_parity_fix_matches_round_pm1_brute_force]),
    ("parity fix dropped", "    if (sum & 1) {\n        int j = 0;", "    if (0) {\n        int j = 0;",
     [lambda: P.test_decoder_is_nearest_point_by_brute_force(O.E8)]),
    ("E8 keeps the farther candidate", "(dB < dA) ? B : A", "(dB > dA) ? B : A",
     [lambda: P.test_decoder_is_nearest_point_by_brute_force(O.E8)]),
    ("A2 point uses sqrt(3) for sqrt(3)/2", "p[1] = (float)q[1] * HQREF_SQRT3_2;", "p[1] = (float)q[1] * HQREF_SQRT3;",
     [lambda: P.test_decoder_is_nearest_point_by_brute_force(O.A2)]),
    ("E8 implied parity not restored", "mm[7] = 2 * m[7] + (s & 1);", "mm[7] = 2 * m[7];",
     [lambda: P.test_strip_reinsert_roundtrip_and_bits_removed(O.E8)]),
    ("zigzag off by one", "return m >= 0 ? 2u * (uint32_t)m :", "return m >= 0 ? 2u * (uint32_t)m + 1u :",
     [P.test_zigzag_published_table]),
    ("inverse scale uses sqrt(127)", "(1.0 / ((double)alpha * sqrt(128.0)))", "(1.0 / ((double)alpha * sqrt(127.0)))",
     [P.test_dithered_reconstruction_is_unbiased_regression]),
    ("inverse drops the sign diagonal", "out[i] = (hqref_sign(seed, sign_col0 + (uint64_t)i) < 0) ? -v[i] : v[i];",
     "out[i] = v[i];", [lambda: P.test_roundtrip_error_within_covering_bound(O.E8)]),
    ("dither uniform from the wrong bits", "(uint32_t)(h >> 40)", "(uint32_t)(h >> 41)",
     [P.test_dither_uniform_follows_published_generator]),
    ("dither box too small", "case HQREF_E8: return 4.0f;", "case HQREF_E8: return 2.0f;",
     [lambda: P.test_subtractive_dither_error_is_uniform_on_voronoi_cell(O.E8, "E8", "2E8")]),
    ("generator increment starts at i", "(i + 1u) * 0x9E3779B97F4A7C15ull", "i * 0x9E3779B97F4A7C15ull",
     [P.test_splitmix64_published_vectors]),
    ("Rice unary drops a bit of the quotient",
     "pos += z[i] >> hqref_symbol_k(lat, k, dk_last, (int)(i % n));\n            put_bit(un, pos++, 1);",
     "pos += z[i] >> (hqref_symbol_k(lat, k, dk_last, (int)(i % n)) + 1);\n            put_bit(un, pos++, 1);",
     [lambda: P.test_chunk_planes_roundtrip_and_same_bits_as_concatenated(O.E8, 2)]),
    ("forward rotation uses Q transposed", "acc = fmaf(Q[i * 128 + j], x[j], acc);",
     "acc = fmaf(Q[j * 128 + i], x[j], acc);", [PR.test_rotation_of_basis_vectors_is_exact]),
    ("inverse rotation not transposed", "acc = fmaf(Q[i * 128 + j], z[i], acc);",
     "acc = fmaf(Q[j * 128 + i], z[i], acc);",
     [PR.test_rotation_of_basis_vectors_is_exact, lambda: PR.test_rotated_roundtrip_error_within_covering_bound(O.E8)]),
    ("rotated inverse scale keeps the Hadamard 1/sqrt(128)",
     "float hqref_scale_inv_rot(float alpha) { return (float)(1.0 / (double)alpha); }",
     "float hqref_scale_inv_rot(float alpha) { return (float)(1.0 / ((double)alpha * sqrt(128.0))); }",
     [PR.test_rotated_dithered_reconstruction_is_unbiased_regression]),
    ("Box-Muller radius loses its factor 2", "return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);",
     "return sqrt(-log(u1)) * cos(two_pi * u2);", [PR.test_gaussian_draws_are_standard_normal]),
    ("last symbol keeps the full Rice parameter", "if (n > 1 && i == n - 1) return (k > dk_last) ? k - dk_last : 0;",
     "if (n > 1 && i == n - 1) return k;",
     [PK.test_symbol_k_follows_the_definition, lambda: PK.test_two_k_planes_hold_the_textbook_codewords(O.E8, 2, 1)]),
    ("first symbol of the block takes the reduced parameter", "if (n > 1 && i == n - 1) return",
     "if (n > 1 && i == 0) return", [lambda: PK.test_two_k_planes_hold_the_textbook_codewords(O.D4, 2, 1)]),
    ("remainders at i * k_i instead of the running sum",
     "for (int b = 0; b < ki; b++) put_bit(rem, rpos++, (z[i] >> b) & 1u);",
     "for (int b = 0; b < ki; b++) put_bit(rem, (uint64_t)i * (uint64_t)ki + (uint64_t)b, (z[i] >> b) & 1u);",
     [lambda: PK.test_two_k_planes_hold_the_textbook_codewords(O.A2, 2, 1)]),
    ("int8 range counts 128 as fitting", "if (v < -128 || v > 127) *overflow += 1;",
     "if (v < -128 || v > 128) *overflow += 1;",
     [PG.test_code_range_definition, lambda: PG.test_range_of_constant_tiles_is_closed_form(O.E8)]),
    ("int8 range counts -128 as overflow", "if (v < -128 || v > 127) *overflow += 1;",
     "if (v <= -128 || v > 127) *overflow += 1;",
     [PG.test_code_range_definition, lambda: PG.test_range_of_alternating_tiles_is_closed_form(O.Z, 2)]),
    ("range taken over the stripped symbols", "            hqref_code_range(q, 128, max_abs, overflow);",
     "            { int32_t m[128]; uint32_t cs; for (int b = 0; b < 128; b += hqref_lattice_dim(lat))"
     " hqref_strip(lat, q + b, m + b, &cs); hqref_code_range(m, 128, max_abs, overflow); }",
     [lambda: PG.test_range_of_constant_tiles_is_closed_form(O.E8)]),
    ("weights dither counter ignores the row", "*e0 = (uint64_t)(r * t->cols + tc * 128);",
     "*e0 = (uint64_t)(tc * 128);", [PG.test_weights_dither_counter_is_row_major_element_index]),
    ("Gaussian radius from one bit too few", "double u1 = ((double)(h >> 32) + 0.5) * 0x1p-32;",
     "double u1 = ((double)(h >> 33) + 0.5) * 0x1p-32;", [PR.test_gaussian_draws_are_standard_normal]),
]


@pytest.mark.parametrize("name,find,repl,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, find, repl, pins):
    src = O.source()
    assert src.count(find) == 1, f"mutation anchor not unique: {find!r}"
    path = O.build_variant(src.replace(find, repl), str(tmp_path / "libhqref_variant.so"))
    caught = []
    with O.using_library(path):
        for pin in pins:
            try:
                pin()
            except AssertionError:
                caught.append(True)
            except ValueError:      # the oracle's own corruption check also counts
                caught.append(True)
    assert caught, f"no pin caught: {name}"
