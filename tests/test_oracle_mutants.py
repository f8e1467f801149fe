"""Plant plausible mistakes in a copy of the oracle's C source and check that
the pins catch every one (CPU only).  The real oracle is never modified."""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

# (name, exact text in attn_oracle.c, replacement)
MUTANTS = [
    ("dropped_scale", "s[j] = scale * acc;", "s[j] = acc;"),
    ("exp_sign_flipped", "z += exp(s[j] - m);", "z += exp(m - s[j]);"),
    ("lse_missing_max", "const double l = m + log(z);\n    for (int t = 0; t < d; ++t) o[t] = 0.0;",
     "const double l = log(z);\n    for (int t = 0; t < d; ++t) o[t] = 0.0;"),
    ("weights_not_normalised", "const double w = exp(s[j] - l);", "const double w = exp(s[j] - m);"),
    ("key_index_frozen", "const double *kj = k + j * (int64_t)d;", "const double *kj = k;"),
    ("value_from_key", "const double *vj = v + j * (int64_t)d;", "const double *vj = k + j * (int64_t)d;"),
    ("causal_off_by_one", "int64_t n = i + (Skv - Sq) + 1;", "int64_t n = i + (Skv - Sq);"),
    ("causal_top_left", "int64_t n = i + (Skv - Sq) + 1;", "int64_t n = i + 1;"),
    ("gqa_modulo_map", "const int64_t g = h / group;\n                const double *kh = k + ((b * Hkv + g) * (int64_t)Skv) * d;\n                const double *vh = v + ((b * Hkv + g) * (int64_t)Skv) * d;\n                attn_one_row(q + r * d",
     "const int64_t g = h % Hkv;\n                const double *kh = k + ((b * Hkv + g) * (int64_t)Skv) * d;\n                const double *vh = v + ((b * Hkv + g) * (int64_t)Skv) * d;\n                attn_one_row(q + r * d"),
    ("split_chunk_floor", "const int64_t cs = (L + num_splits - 1) / num_splits;",
     "const int64_t cs = L / num_splits + 1;"),
    ("combine_weight_uses_max", "const double w = exp(ls[c] - l);", "const double w = exp(ls[c] - m);"),
    ("combine_lse_missing_max", "const double l = m + log(z);\n        for (int c = 0;",
     "const double l = log(z);\n        for (int c = 0;"),
    ("decode_reads_lmax", "attn_one_row(q + r * d, kh, vh, seqlens[b],", "attn_one_row(q + r * d, kh, vh, Lmax,"),
    ("aligned_chunk_rounds_down", "const int64_t cs = (cs0 + align - 1) / align * align;",
     "const int64_t cs = cs0 / align * align;"),
    ("aligned_chunk_ignores_align", "const int64_t cs = (cs0 + align - 1) / align * align;",
     "const int64_t cs = cs0;"),
    ("bwd_drops_softmax_jacobian_term", "const double ds = p[j] * (dp[j] - dsum);",
     "const double ds = p[j] * dp[j];"),
    ("bwd_dk_missing_scale", "dkh[j * d + t] += scale * ds * qi[t];", "dkh[j * d + t] += ds * qi[t];"),
    ("bwd_dv_uses_dp", "dvh[j * d + t] += p[j] * doi[t];", "dvh[j * d + t] += dp[j] * doi[t];"),
    ("bwd_dq_uses_query", "dqi[t] += scale * ds * kh[j * d + t];", "dqi[t] += scale * ds * qi[t];"),
    ("e4m3_bias_8", "mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_subnormal_implicit_one", "mag = ldexp((double)m / 8.0, -6);",
     "mag = ldexp(1.0 + (double)m / 8.0, -6);"),
    ("e4m3_nan_code_missed", "if (e == 15 && m == 7)\n        return NAN;",
     "if (e == 16 && m == 7)\n        return NAN;"),
    ("e4m3_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
    ("dequant_query_head_modulo", "const int64_t g = h / group;\n            const double f",
     "const int64_t g = h % Hkv;\n            const double f"),
    ("dequant_batch_ignored", "descale[b * Hkv + g]", "descale[g]"),
    ("gelu_missing_half", "return 0.5 * h * (1.0 + erf(h / sqrt(2.0)));",
     "return h * (1.0 + erf(h / sqrt(2.0)));"),
    ("gelu_erf_unscaled", "return 0.5 * h * (1.0 + erf(h / sqrt(2.0)));",
     "return 0.5 * h * (1.0 + erf(h));"),
    ("ffn_w1_row_frozen", "const double *w = w1 + (int64_t)f * D;", "const double *w = w1;"),
    ("ffn_w2_row_frozen", "const double *w = w2 + (int64_t)i * F;", "const double *w = w2;"),
    ("ffn_token_frozen", "ffn_token_hidden(x + t * D, w1, D, F, hid);",
     "ffn_token_hidden(x, w1, D, F, hid);"),
    ("ffn_hidden_token_frozen", "ffn_token_hidden(x + t * D, w1, D, F, hid + t * F);",
     "ffn_token_hidden(x, w1, D, F, hid + t * F);"),
    ("ffn_hidden_no_gelu", "hid[f] = gelu(acc);", "hid[f] = acc;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not unique/absent"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = str(tmp_path / "mutant.so")
    oracle.build(str(src), so, force=True)
    lib = oracle.load(so)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError) as e:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
