"""Mutation check of the oracle's pins, entirely on the CPU.

Each case copies the oracle's C source, plants one plausible mistake (a swapped sign
mapping, a wrong bit or group index, a dropped term, a transposed operand, ...), builds
the copy with gcc into a temporary directory and runs every pin from
``test_oracle_pins.py`` against it. The case passes when at least one pin fails, i.e.
the pins would have caught that mistake in the real oracle.
"""

import os
import shutil

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    "sign_mapping_swapped": (
        "return bit ? s : -s;", "return bit ? -s : s;"),
    "bit_order_msb_first": (
        "uint32_t bit = (words[n * (K / 32) + k / 32] >> (k % 32)) & 1u;",
        "uint32_t bit = (words[n * (K / 32) + k / 32] >> (31 - k % 32)) & 1u;"),
    "group_index_64": (
        "double s = bqo_f16_to_f64(scales[n * (K / 128) + k / 128]);",
        "double s = bqo_f16_to_f64(scales[n * (K / 128) + (k / 64) % (K / 128)]);"),
    "scale_row_index": (
        "double s = bqo_f16_to_f64(scales[n * (K / 128) + k / 128]);",
        "double s = bqo_f16_to_f64(scales[k / 128]);"),
    "ternary_code_map_reversed": (
        "return s * (double)((int)code - 1);", "return s * (double)(1 - (int)code);"),
    "ternary_field_shift": (
        "uint32_t code = (words[n * (K / 16) + k / 16] >> (2 * (k % 16))) & 3u;\n    if (code == 3)",
        "uint32_t code = (words[n * (K / 16) + k / 16] >> (2 * (15 - k % 16))) & 3u;\n    if (code == 3)"),
    "scale_dropped": (
        "acc += xv * bqo_weight(fmt, words, scales, K, n, k);",
        "acc += xv * (bqo_weight(fmt, words, scales, K, n, k) > 0 ? 1.0 : -1.0);"),
    "x_transposed": (
        "double xv = x_value(x, xt, m * K + k);", "double xv = x_value(x, xt, k * M + m);"),
    "bound_uses_y": (
        "bound[m * R + r] = 2e-3 * mag;", "bound[m * R + r] = 2e-3 * fabs(acc);"),
    "pack_bit_offset": (
        "words[n * W + k / 32] |= (uint32_t)1 << (k % 32);",
        "words[n * W + k / 32] |= (uint32_t)1 << ((k + 1) % 32);"),
    "pack_ternary_wrong_code": (
        "uint32_t code = (uint32_t)(v + 1);", "uint32_t code = (uint32_t)(1 - v);"),
    "unpack_misses_code3": (
        "if (code == 3) {\n                bad++;", "if (code == 4) {\n                bad++;"),
    "f16_exponent_off": (
        "v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    "f16_subnormal_as_normal": (
        "v = ldexp((double)f, -24);", "v = ldexp((double)(1024 + f), -25);"),
    "bf16_round_9_bits": (
        "double r = round_to_format(v, 8, -126,", "double r = round_to_format(v, 9, -126,"),
    "embed_wrong_row": (
        "out[t * K + k] = bqo_weight(fmt, words, scales, K, id, k);",
        "out[t * K + k] = bqo_weight(fmt, words, scales, K, t % N, k);"),
    "mlx_bias_sign": (
        "uint16_t bias = bqo_f64_to_f16(-s);", "uint16_t bias = bqo_f64_to_f16(s);"),
    "b3_codes_lsb_first": (
        "int8_t w = q[n * K + 128 * g + b3_first(j) + p];",
        "int8_t w = q[n * K + 128 * g + b3_first(j) + (cnt - 1 - p)];"),
    "b3_encode_floor": (
        "return (uint8_t)((256 * v + kPow3[n] - 1) / kPow3[n]);",
        "return (uint8_t)((256 * v) / kPow3[n]);"),
    "b3_four_code_bytes_in_group": (
        "return 26 * first + 24 * nb + 2 * (g - first) + (j - 24);",
        "return 26 * first + 26 * (g - first) + j;"),
    "b3_digit_order": (
        "return (int)((v / kPow3[n - 1 - p]) % 3);", "return (int)((v / kPow3[p]) % 3);"),
    "b3_every_byte_valid": (
        "*valid = b3_encode(v, n) == byte;", "*valid = 1;"),
    "b3_decode_rounds": (
        "int64_t v = ((int64_t)byte * kPow3[n]) / 256;",
        "int64_t v = ((int64_t)byte * kPow3[n] + 128) / 256;"),
    "topk_ties_high_index_first": (
        "return va > vb || (va == vb && ia < ib);", "return va > vb || (va == vb && ia > ib);"),
    "sample_temperature_multiplies": (
        "p[i] = exp((vals[i] - vals[0]) / T);", "p[i] = exp((vals[i] - vals[0]) * T);"),
    "sample_top_p_strict": (
        "if (c >= top_p)", "if (c > top_p)"),
    "sample_not_renormalised": (
        "cum += p[i] / kept;", "cum += p[i] / z;"),
    "quantize_zero_group_full_support": (
        "if (score > best) {", "if (score >= best) {"),
    "quantize_tie_takes_larger_support": (
        "if (score > best) {", "if (score > best || (score == best && score > 0.0)) {"),
    "quantize_sort_ascending": (
        "return a->a > b->a ? -1 : 1;", "return a->a > b->a ? 1 : -1;"),
    "quantize_binary_scale_127": (
        "s[n * (K / 128) + g] = bqo_f64_to_f16(sum / 128.0);", "s[n * (K / 128) + g] = bqo_f64_to_f16(sum / 127.0);"),
    "quantize_binary_zero_negative": (
        "qg[k] = wg[k] >= 0.0f ? 1 : -1;\n                    sum +=", "qg[k] = wg[k] > 0.0f ? 1 : -1;\n                    sum +="),
    "mlp_silu_sign": (
        "a[m * F + f] = g / (1.0 + exp(-g)) * u;", "a[m * F + f] = g / (1.0 + exp(g)) * u;"),
    "mlp_gate_up_swapped": (
        "a[m * F + f] = g / (1.0 + exp(-g)) * u;", "a[m * F + f] = u / (1.0 + exp(-u)) * g;"),
    "mlp_bound_gate_scale": (
        "mag += fabs(av * bqo_f16_to_f64(sd[n * (F / 128) + j / 128]));",
        "mag += fabs(av * bqo_f16_to_f64(sg[(n % F) * (K / 128)]));"),
    "sum_skips_last_k": (
        "for (int64_t k = 0; k < K; k++) {\n                double xv",
        "for (int64_t k = 0; k < K - 1; k++) {\n                double xv"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = os.path.join(os.path.dirname(oracle.__file__), "bq_oracle.c")
    text = open(src).read()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    mdir = tmp_path / name
    mdir.mkdir()
    shutil.copy(os.path.join(os.path.dirname(src), "bq_oracle.h"), mdir / "bq_oracle.h")
    (mdir / "bq_oracle.c").write_text(text.replace(old, new))
    lib = oracle.build(force=True, src=str(mdir / "bq_oracle.c"), out=str(mdir / "libmut.so"))
    mutant = oracle.Oracle(lib)
    failed = []
    for pin in pins.PINS:
        try:
            pin(mutant)
        except Exception as e:  # an assertion or an error both count as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin catches mutant {name}"
