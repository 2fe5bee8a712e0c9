"""Plant a plausible mistake in a copy of the oracle's C source and check that
at least one pin fails on it (CPU only). A pin set that passes a mutant would
not protect the oracle against that mistake."""
import os
import shutil

import pytest

import helpers
import oracle as O
import oracle_pins as P

# (name, text in qfp4_oracle.c, replacement)
MUTATIONS = [
    ("fwht_butterfly_sign", "w[j + h] = a - b;", "w[j + h] = b - a;"),
    ("sign_flip_dropped", "if ((sign_bits >> j) & 1u) w[j] = -w[j];", "if (0) w[j] = -w[j];"),
    ("rotation_norm", "(float)(1.0 / sqrt((double)nh))", "(float)(1.0 / (double)nh)"),
    ("rtn_tie_to_odd", "if (d < best || (d == best && (j % 2) == 0)) {\n                best = d;\n                idx = j;",
     "if (d < best || (d == best && (j % 2) == 1)) {\n                best = d;\n                idx = j;"),
    ("e4m3_bias", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    ("nvfp4_tensor_scale", "s_enc = 2688.0f / amax;", "s_enc = 2048.0f / amax;"),
    ("nvfp4_block_top", "float d = amax_b / 6.0f;", "float d = amax_b / 4.0f;"),
    ("mxfp4_exponent_offset", "int E = floor_log2f(amax_b) - 2;", "int E = floor_log2f(amax_b) - 1;"),
    ("mxfp4_ru_floor_rule", "while ((double)amax_b > 6.0 * ldexp(1.0, E)) E += 1;",
     "while ((double)amax_b >= 8.0 * ldexp(1.0, E)) E += 1;"),
    ("mxfp4_ru_not_strict", "while ((double)amax_b > 6.0 * ldexp(1.0, E)) E += 1;",
     "while ((double)amax_b >= 6.0 * ldexp(1.0, E)) E += 1;"),
    ("sr_compare_flipped", "idx = (rho < p) ? lo + 1 : lo;", "idx = (rho > p) ? lo + 1 : lo;"),
    ("philox_multiplier", "(uint64_t)0xD2511F53u", "(uint64_t)0xD2511F55u"),
    ("philox_key_bump", "k1 += 0xBB67AE85u;", "k1 += 0xBB67AE86u;"),
    ("quartet2_alpha_inverted", "alpha = (den == 0.0f) ? 1.0f : num / den;", "alpha = (den == 0.0f) ? 1.0f : den / num;"),
    ("tree_sum_wrong_term", "s[j] = s[j] + s[j + stride];", "s[j] = s[j] + s[j + stride / 2];"),
    ("dot_tree_first_stride_term", "s[j] = fmaf(a[j], b[j], a[j + h] * b[j + h]);",
     "s[j] = fmaf(a[j], b[j], a[j + h] * b[j]);"),
    ("dot_tree_half_dropped", "return tree_sum(s, h);", "return tree_sum(s, h / 2);"),
    ("nibble_order", "out[j / 2] = (uint8_t)(q[j] | (q[j + 1] << 4));", "out[j / 2] = (uint8_t)(q[j + 1] | (q[j] << 4));"),
    ("col_orientation", "for (int64_t j = 0; j < k; ++j) seg[j] = bf16_to_f32(x[j * ld + row]);",
     "for (int64_t j = 0; j < k; ++j) seg[j] = bf16_to_f32(x[(j ^ 1) * ld + row]);"),
    ("scale_sr_always_down", "return (uint8_t)((rho < p) ? lo + 1 : lo);", "return (uint8_t)lo;"),
    ("element_uniform_half", "return (float)((w >> (16u * (uint32_t)(i & 1u))) & 0xFFFFu) * 0x1p-16f;",
     "return (float)(w & 0xFFFFu) * 0x1p-16f;"),
    ("element_uniform_word", "const uint32_t w = random_word(seed, TAG_ELEMENT, stream, i >> 1);",
     "const uint32_t w = random_word(seed, TAG_ELEMENT, stream, i >> 2);"),
    ("element_sr_index", "const uint64_t i = (uint64_t)(r * k + b * nb + j);", "const uint64_t i = (uint64_t)(r * k + b * nb);"),
    ("e8m0_sr_compare_flipped", "    if (rho < p) e += 1;\n", "    if (rho > p) e += 1;\n"),
    ("e8m0_sr_probability", "float p = (t - lo) / lo; /* exact: t in [lo, 2 lo) */",
     "float p = (t - lo) / (2.0f * lo); /* exact: t in [lo, 2 lo) */"),
]


@pytest.fixture(scope="module")
def tmpdir_mut():
    d = helpers.scratch_dir("oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutant_is_caught(name, old, new, tmpdir_mut):
    src = open(os.path.join(os.path.dirname(O.__file__), "qfp4_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(tmpdir_mut, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = O.compile_source(path, os.path.join(tmpdir_mut, f"lib{name}.so"))
    failed = None
    with O.using(lib):
        for check in P.ALL_CHECKS:
            try:
                check()
            except (AssertionError, ValueError) as e:  # noqa: PERF203
                failed = check.__name__
                break
    assert failed is not None, f"no pin catches mutation {name}"
