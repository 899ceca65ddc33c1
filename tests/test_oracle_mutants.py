"""Plant one mistake at a time in a copy of the oracle and check that the pins catch it.

Each mutant is the oracle's C source with one plausible error edited in (a
dropped term, a wrong sign, a wrong index, a transposed operand, a wrong
exponent bias), compiled to a temporary library on the CPU.  The real oracle
is untouched.
"""

import os
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "q4_0_drop_minus_8": ("w[i] = (float)(d * (double)(lo - 8));", "w[i] = (float)(d * (double)(lo));"),
    "q4_0_swap_nibbles": ("int lo = b[2 + i] & 15;\n        int hi = b[2 + i] >> 4;",
                          "int hi = b[2 + i] & 15;\n        int lo = b[2 + i] >> 4;"),
    "q8_0_unsigned": ("int q = (int8_t)b[2 + i];", "int q = (uint8_t)b[2 + i];"),
    "q4_k_min_sign": ("(double)qlo - dmin * (double)m0", "(double)qlo + dmin * (double)m0"),
    "q4_k_scale_index": ("*sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);",
                         "*sc = (s[j + 4] & 15) | ((s[j] >> 6) << 4);"),
    "q4_k_min_high_bits": ("*m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);", "*m = (s[j + 4] >> 4);"),
    "q4_k_group_halves": ("int qlo = qs[32 * g + l] & 15;\n            int qhi = qs[32 * g + l] >> 4;",
                          "int qlo = qs[32 * g + l] >> 4;\n            int qhi = qs[32 * g + l] & 15;"),
    "q4_k_dmin_is_d": ("double dmin = lwq_oracle_f16(rd16(b + 2));\n    const uint8_t *s = b + 4;\n    const uint8_t *qs",
                       "double dmin = lwq_oracle_f16(rd16(b));\n    const uint8_t *s = b + 4;\n    const uint8_t *qs"),
    "q5_k_dmin_is_d": ("double dmin = lwq_oracle_f16(rd16(b + 2));\n    const uint8_t *s = b + 4, *qh",
                       "double dmin = lwq_oracle_f16(rd16(b));\n    const uint8_t *s = b + 4, *qh"),
    "q6_k_no_offset": ("(double)sc[e / 16] * (double)(q - 32)", "(double)sc[e / 16] * (double)(q)"),
    "q6_k_high_shift": ("int high = (qh[32 * n + l] >> (2 * g)) & 3;", "int high = (qh[32 * n + l] >> g) & 3;"),
    "q6_k_low_quarter": ("ql[64 * n + 32 * (g & 1) + l] >> (4 * (g >> 1))", "ql[64 * n + 32 * (g >> 1) + l] >> (4 * (g & 1))"),
    "q6_k_scale_per_32": ("(double)sc[e / 16] * (double)(q - 32)", "(double)sc[e / 32] * (double)(q - 32)"),
    "q6_k_d_offset": ("double d = lwq_oracle_f16(rd16(b + 208));", "double d = lwq_oracle_f16(rd16(b + 206));"),
    "q6_k_unsigned_scale": ("const int8_t *sc = (const int8_t *)(b + 192);", "const uint8_t *sc = (const uint8_t *)(b + 192);"),
    "q5_k_fifth_bit_index": ("(((qh[l] >> (2 * g + h)) & 1) << 4)", "(((qh[l] >> (g + 4 * h)) & 1) << 4)"),
    "q5_k_no_fifth_bit": ("| (((qh[l] >> (2 * g + h)) & 1) << 4)", ""),
    "q5_k_swapped_arrays": ("*qh = b + 16, *qs = b + 48;", "*qh = b + 144, *qs = b + 16;"),
    "q5_k_min_sign": ("(double)q - dmin * (double)m);\n    }\n}\n\nstatic void decode_q2_k",
                      "(double)q + dmin * (double)m);\n    }\n}\n\nstatic void decode_q2_k"),
    "q2_k_min_nibble": ("m = s[e / 16] >> 4;", "m = s[e / 16] & 15;"),
    "q2_k_field_shift": ("int q = (qs[32 * n + l] >> (2 * j)) & 3;", "int q = (qs[32 * n + l] >> j) & 3;"),
    "q2_k_d_is_dmin": ("double d = lwq_oracle_f16(rd16(b + 80));", "double d = lwq_oracle_f16(rd16(b + 82));"),
    "q2_k_half_stride": ("int q = (qs[32 * n + l] >> (2 * j)) & 3;", "int q = (qs[16 * n + l] >> (2 * j)) & 3;"),
    "attn_no_scale": ("s[j] = scale * dot;", "s[j] = dot;"),
    "attn_no_max": ("s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
    "attn_gqa_modulo": ("long b = bh / H, h = bh % H, g = h / G;", "long b = bh / H, h = bh % H, g = h % Hkv;"),
    "attn_values_are_keys": ("const uint16_t *vb = v + (b * Hkv + g) * Lmax * D;",
                             "const uint16_t *vb = k + (b * Hkv + g) * Lmax * D;"),
    "attn_mean_not_softmax": ("out[(b * H + h) * D + d] = acc / sum;", "out[(b * H + h) * D + d] = acc / (double)n;"),
    "attn_ignores_len": ("long n = len[b];", "long n = Lmax;"),
    "attn_den_no_abs": ("acc_abs += s[j] * fabs(vd);", "acc_abs += s[j] * vd;"),
    "f16_bias": ("v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    "f16_subnormal": ("v = ldexp((double)f, -24);", "v = ldexp((double)(1024 + f), -24);"),
    "bf16_bias": ("v = ldexp((double)(128 + f), e - 134);", "v = ldexp((double)(128 + f), e - 133);"),
    "den_no_abs": ("acc_abs += fabs(p);", "acc_abs += p;"),
    "transposed_x": ("xd[i] = act_value(act, x, i);", "xd[i] = act_value(act, x, (i % K) * M + i / K);"),
    "skip_last_k": ("for (long k = 0; k < K; k++) {\n        double p", "for (long k = 0; k + 1 < K; k++) {\n        double p"),
    "sampled_wrong_row": ("lwq_oracle_dequant_row(fmt, Wq + ns[i] * rb, K, w);",
                          "lwq_oracle_dequant_row(fmt, Wq + ms[i] * rb, K, w);"),
}


@pytest.fixture(scope="module")
def src():
    with open(os.path.join(os.path.dirname(oracle.__file__), "lwq_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, src, name):
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *oracle.CFLAGS, str(path), "-o", str(so), "-lm"], check=True)
    lib = oracle.load(str(so))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception as e:  # a crash or a refused call also counts as a detection
            caught.append(f"{pin.__name__}:{type(e).__name__}")
    assert caught, f"no pin catches mutant {name}"
