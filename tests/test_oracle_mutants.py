"""Plausible mistakes planted in copies of the oracle (on the CPU) must each fail a pin.

Each mutant is the oracle's C source with one textual change, compiled into a temporary
library; the pins of oracle_pins.py then run against it and at least one must fail. This
shows the pins are strong enough that a dropped term, a wrong sign, index or operand in the
oracle would not go unnoticed.
"""
import os

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "sdpa_oracle.c")

MUTANTS = {
    "causal_off_by_one": ("!(j <= off + i)", "!(j < off + i)"),
    "gqa_interleaved_heads": ("? (h / group) :", "? (h % Hkv) :"),
    "bottom_right_sign": ("off = kvlen_b - qlen_b;", "off = qlen_b - kvlen_b;"),
    "scale_dropped": ("double x = scale * dot;", "double x = dot;"),
    "kv_length_inclusive": ("int ok = (j < kvlen_b);", "int ok = (j <= kvlen_b);"),
    "q_length_inclusive": ("if (i >= qlen_b) {", "if (i > qlen_b) {"),
    "mask_strides_swapped": ("p->mask[j * p->mask_stride[0] + i * p->mask_stride[1]",
                             "p->mask[i * p->mask_stride[0] + j * p->mask_stride[1]"),
    "bias_sign": ("      x += p->bias[", "      x -= p->bias["),
    "bias_scaled": ("    s[j] = x;\n", "    s[j] = x * 0.5 + 0.5 * scale * dot;\n"),
    "not_normalised": ("const double w = s[j] / denom;", "const double w = s[j];"),
    "empty_row_zero": ("o[e] = NAN;", "o[e] = 0.0;"),
    "default_scale_dv": ("1.0 / sqrt((double)D)", "1.0 / sqrt((double)Dv)"),
    "value_head_wrong": ("const double* vj = v + ((b * Lk + j) * Hkv + g) * Dv;",
                         "const double* vj = v + ((b * Lk + j) * Hkv + (g + 1) % Hkv) * Dv;"),
    "cache_rows_reversed": ("index[b] + t) * row", "index[b] + n_new - 1 - t) * row"),
    "block_class_swapped": ("(set == cells ? 2 : 1)", "(set == cells ? 1 : 2)"),
    "block_bits_reversed": ("word |= (1u << c);", "word |= (1u << (31 - c));"),
    "block_full_at_edge": ("(set == cells ? 2 : 1)", "(set == bq * bk ? 2 : 1)"),
    "rope_pairs_adjacent": ("const double x0 = xr[c], x1 = xr[c + half];", "const double x0 = xr[c], x1 = xr[(c + 1) % d];"),
    "rope_sin_sign": ("o[c] = x0 * cos(a) - x1 * sin(a);", "o[c] = x0 * cos(a) + x1 * sin(a);"),
    "rope_frequency_exponent": ("pow(base, -2.0 * (double)c / (double)d)", "pow(base, -1.0 * (double)c / (double)d)"),
    "weights_dropout_unscaled": ("? w / (1.0 - drop_p) : 0.0", "? w : 0.0"),
    "lse_without_max": ("  if (lse) *lse = m + log(denom);", "  if (lse) *lse = log(denom);"),
    "weights_dropout_inverted": ("dropout_keep(seed, base + (uint64_t)j, thr) ?", "!dropout_keep(seed, base + (uint64_t)j, thr) ?"),
    "weights_dropout_same_draw_per_group": ("0x9e3779b97f4a7c15ULL);\n  const uint32_t u = (uint32_t)(r >> (16 * (index & 3)))",
                                            "0x9e3779b97f4a7c15ULL);\n  const uint32_t u = (uint32_t)(r >> 0)"),
    "weights_head_batch_swapped": ("double* wrow = weights + ((b * H + h) * Lq + i) * Lk;",
                                   "double* wrow = weights + ((h * B + b) * Lq + i) * Lk;"),
    "backward_delta_sign": ("x[j] * (dw[j] - wdw)", "x[j] * (dw[j] + wdw)"),
    "backward_dk_unscaled": ("dkj[c] += scale * dx * qi[c];", "dkj[c] += dx * qi[c];"),
    "backward_dv_from_dx": ("dvj[e] += x[j] * doi[e];", "dvj[e] += dx * doi[e];"),
    "backward_dscale_scaled": ("total += dx * dot;", "total += dx * dot * scale;"),
    "backward_causal_off_by_one": ("          if (p->causal != 0 && !(j <= off + i)) a = 0;",
                                   "          if (p->causal != 0 && !(j < off + i)) a = 0;"),
    "weights_causal_off_by_one": ("      if (p->causal != 0 && !(j <= off + i)) a = 0;",
                                  "      if (p->causal != 0 && !(j < off + i)) a = 0;"),
    # packed mutants move starts only toward lower addresses, so every access stays in bounds
    "packed_kv_segments_ignored": ("kv_segments ? kv_segments : q_segments;", "q_segments;"),
    "packed_query_start": ("q + q0 * H * p->dqk", "q + q0 * Hkv * p->dqk"),
    "packed_key_start": ("k + k0 * Hkv * p->dqk", "k + k0 * p->dqk"),
    "packed_out_start": ("out + q0 * H * p->dv", "out + q0 * Hkv * p->dv"),
    "packed_first_offset_only": ("p->q_offset ? p->q_offset + s", "p->q_offset ? p->q_offset"),
    "packed_kv_lengths_first_only": ("p->kv_lengths ? p->kv_lengths + s", "p->kv_lengths ? p->kv_lengths"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = oracle.load(oracle.build(str(mutated), str(tmp_path / "libmutant.so"), force=True))
    failed = []
    for p in PINS:
        try:
            p(lib)
        except Exception as e:  # noqa: BLE001 — any failure counts
            failed.append(p.__name__)
    assert failed, f"mutant {name} passed every pin"
