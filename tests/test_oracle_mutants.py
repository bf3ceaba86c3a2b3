"""Plant plausible mistakes in copies of the C oracle and check that the pins
catch every one of them (each mutant must fail at least one pin).

The mutants are textual edits of bitlinear_oracle.c compiled into a temporary
directory; the real oracle is never modified. Each edit names a mistake a
careful reader could make: a dropped term, a wrong sign or index, a
transposed operand, a different rounding mode or constant, a swapped bit
position in the packed layout.
"""
import os
import tempfile

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "bitlinear_oracle.c")

MUTANTS = {
    "weight_round_half_away": ("rintf(W[i] / gamma)", "roundf(W[i] / gamma)"),
    "act_round_half_away": ("rintf(row[k] * scale)", "roundf(row[k] * scale)"),
    "gamma_without_abs": ("sum += fabs((double)W[i]);", "sum += (double)W[i];"),
    "gamma_mean_off_by_one": ("sum / (double)count", "sum / (double)(count - 1)"),
    "beta_without_abs": ("float a = fabsf(row[k]);", "float a = row[k];"),
    "weight_clip_at_two": ("if (q > 1.0f)", "if (q > 2.0f)"),
    "weight_scale_multiplies": ("rintf(W[i] / gamma)", "rintf(W[i] * gamma)"),
    "qb_is_128": ("const float scale = ORACLE_QB / b;", "const float scale = 128.0f / b;"),
    "epsilon_1e_3": ("ORACLE_EPS = 1e-5f", "ORACLE_EPS = 1e-3f"),
    "matmul_transposed_weight": ("(int64_t)Wq[n * K + k];", "(int64_t)Wq[k * N + n];"),
    "matmul_subtracts": ("s += (int64_t)xq[m * K + k]", "s -= (int64_t)xq[m * K + k]"),
    "matmul_skips_last_k": ("for (int64_t k = 0; k < K; ++k)\n                s += (int64_t)xq",
                            "for (int64_t k = 0; k + 1 < K; ++k)\n                s += (int64_t)xq"),
    "rescale_drops_gamma": ("(beta[m] * gamma) / ORACLE_QB", "(beta[m]) / ORACLE_QB"),
    "rescale_divides_acc": ("(float)acc[m * N + n] * s", "(float)acc[m * N + n] / s"),
    "bf16_ties_away": ("(dropped == 0x8000u && (kept & 1u))", "(dropped == 0x8000u)"),
    "bf16_truncates": ("kept += 1u;", "kept += 0u;"),
    "bf16_widen_stray_low_bit": ("uint32_t bits = (uint32_t)in[i] << 16;",
                                 "uint32_t bits = ((uint32_t)in[i] << 16) | 0x8000u;"),
    "bf16_widen_shift_15": ("uint32_t bits = (uint32_t)in[i] << 16;",
                            "uint32_t bits = (uint32_t)in[i] << 15;"),
    "bf16_widen_drops_sign": ("uint32_t bits = (uint32_t)in[i] << 16;",
                              "uint32_t bits = ((uint32_t)in[i] & 0x7fffu) << 16;"),
    "pack_swaps_j_b": ("<< (8 * b + 2 * j)", "<< (8 * j + 2 * b)"),
    "pack_code_negated": ("(uint32_t)(v + 1)", "(uint32_t)(1 - v)"),
    "pack_word_index": ("16 * w + 4 * j + b;", "16 * w + 4 * b + j;"),
    "pack_row_stride": ("512 * g + 32 * r + 4 * w", "512 * g + 32 * w + 4 * r"),
    "pack_padding_rows": ("(n < N) ? Wq[n * K + k] : 0", "(n < N) ? Wq[n * K + k] : -1"),
    "b3_digit_order": ("value += (v + 1) * power;", "value = value * 3 + (v + 1);"),
    "b3_stream_transposed": ("const int64_t k = 160 * g + 16 * w + 4 * j + b;",
                             "const int64_t k = 160 * g + 16 * w + 4 * b + j;"),
    "b3_padding_code": ("const int v = (n < N && k < K) ? Wq[n * K + k] : 0;",
                        "const int v = (n < N && k < K) ? Wq[n * K + k] : -1;"),
    "b3_byte_order": ("packed[blk * 16 * row_bytes + 512 * g + 32 * r + B]",
                      "packed[blk * 16 * row_bytes + 512 * g + 32 * r + (31 - B)]"),
    "rms_drops_eps": ("sqrtf(ms + eps)", "sqrtf(ms)"),
    "rms_mean_over_k_minus_1": ("ss / (double)K", "ss / (double)(K - 1)"),
    "rms_forgets_sqrt": ("1.0f / sqrtf(ms + eps)", "1.0f / (ms + eps)"),
    "rms_multiplies_by_rms": ("1.0f / sqrtf(ms + eps)", "sqrtf(ms + eps)"),
    "rms_sum_of_abs": ("ss += v * v;", "ss += fabs(v);"),
    "rms_gain_by_token": ("(row[k] * r) * g[k]", "(row[k] * r) * g[m]"),
    "rms_gain_first": ("(row[k] * r) * g[k]", "(row[k] * g[k]) * r"),
    "rms_gain_dropped": ("(row[k] * r) * g[k]", "(row[k] * r)"),
    "glu_no_relu": ("gate[i] > 0.0f ? gate[i] : 0.0f", "gate[i]"),
    "glu_relu_inverted": ("gate[i] > 0.0f ? gate[i] : 0.0f", "gate[i] < 0.0f ? gate[i] : 0.0f"),
    "glu_no_square": ("(r * r) * up[i]", "r * up[i]"),
    "glu_ignores_up": ("(r * r) * up[i]", "(r * r)"),
    "glu_adds_up": ("(r * r) * up[i]", "(r * r) + up[i]"),
}


def test_unmutated_oracle_passes_every_pin():
    assert pins.failing_pins(oracle.default()) == []


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, f"mutation target not found: {old!r}"
    mutated = source.replace(old, new)
    src = tmp_path / "mutant.c"
    src.write_text(mutated)
    so = oracle.build(str(src), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(oracle.load(so))
    failed = pins.failing_pins(orc)
    assert failed, f"mutant {name} passed every pin"
