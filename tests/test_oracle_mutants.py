"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and runs the pin checks of
test_oracle_pins against that build: at least one pin must fail.  The
committed oracle itself is never modified.
"""
import os
import shutil

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

# (name, exact text in the oracle, planted mistake)
MUTANTS = [
    ("tie_to_higher_index", "keys[e] > keys[best]) best = e;", "keys[e] >= keys[best]) best = e;"),
    ("sigmoid_sign", "return 1.0 / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(v));"),
    ("silu_sign", "return u / (1.0 + exp(-u));", "return u / (1.0 + exp(u));"),
    ("renorm_dropped", "if (c->norm_topk)\n", "if (0 && c->norm_topk)\n"),
    ("gate_from_slot_index", "gates[j] = scores[ids[j]];", "gates[j] = scores[j];"),
    ("down_transposed", "o += elem(wd, w_off_out + (int64_t)i * hid + n, c->dtype) * a[n];",
     "o += elem(wd, w_off_out + (int64_t)n * c->d + i, c->dtype) * a[n];"),
    ("bwd_down_transposed", "s += elem(wd, w_off_out + (int64_t)i * hid + n, c->dtype) * elem(dy",
     "s += elem(wd, w_off_out + (int64_t)n * c->d + i, c->dtype) * elem(dy"),
    ("gate_up_swapped", "a[n] = silu(u) * v;", "a[n] = silu(v) * u;"),
    ("router_transposed", "elem(wr, (int64_t)e * c->d + i, c->dtype)",
     "elem(wr, (int64_t)i * c->E + e, c->dtype)"),
    ("softmax_no_normaliser", "scores[e] = exp(logits[e] - m) / z;",
     "scores[e] = exp(logits[e] - m);"),
    ("permutation_unstable", "for (int64_t r = 0; r < R; ++r)\n            if (ids[r] == e) sorted_rows[pos++]",
     "for (int64_t r = R - 1; r >= 0; --r)\n            if (ids[r] == e) sorted_rows[pos++]"),
    ("offsets_inclusive", "offsets[e + 1] = offsets[e] + counts[e];",
     "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
    ("shared_gate_sign", "*shared_gate = sigmoid(s);", "*shared_gate = sigmoid(-s);"),
    ("gate_weight_dropped", "out[i] += g * o;", "out[i] += o;"),
    ("selection_by_raw_logit_under_sigmoid",
     "keys[e] = (c->score == ORACLE_SIGMOID) ? sigmoid(logits[e]) : logits[e];",
     "keys[e] = (c->score == ORACLE_SIGMOID) ? -logits[e] : logits[e];"),
    ("balance_bias_ignored", "if (bias)\n            keys[e] = scores[e]", "if (0 && bias)\n            keys[e] = scores[e]"),
    ("balance_bias_subtracted", "keys[e] = scores[e] + (double)bias[e];", "keys[e] = scores[e] - (double)bias[e];"),
    ("balance_bias_on_logits", "keys[e] = scores[e] + (double)bias[e];", "keys[e] = logits[e] + (double)bias[e];"),
    ("balance_bias_leaks_into_gates", "gates[j] = scores[ids[j]];", "gates[j] = keys[ids[j]];"),
    ("bias_update_sign", "if (mean > load) sign = 1.0;", "if (mean > load) sign = -1.0;"),
    ("bias_update_mean_over_tokens", "double mean = total / (double)c->E;", "double mean = total / (double)c->T;"),
    ("score_mean_not_divided", "mean[e] = s / (double)c->T;", "mean[e] = s;"),
    ("switch_loss_without_N", "*loss = alpha * (double)c->E * sum;", "*loss = alpha * sum;"),
    ("switch_frac_over_assignments", "(double)counts[e] / (double)c->T", "(double)counts[e] / (double)(c->T * c->k)"),
    ("bwd_dsilu", "return s * (1.0 + u * (1.0 - s));", "return s * (1.0 + u * s);"),
    ("bwd_renorm_dropped", "ds[ids[j]] = c->norm_topk ? (dg[j] - dot) / q : dg[j];", "ds[ids[j]] = dg[j];"),
    ("bwd_softmax_not_centred", "dl[e] = scores[e] * (ds[e] - sd);", "dl[e] = scores[e] * ds[e];"),
    ("bwd_sigmoid_factor", "dl[e] = ds[e] * scores[e] * (1.0 - scores[e]);", "dl[e] = ds[e] * scores[e];"),
    ("bwd_gate_missing", "double da = g * r[n];", "double da = r[n];"),
    ("bwd_dv_uses_dsilu", "double dv = da * silu(u[n]);", "double dv = da * dsilu(u[n]);"),
    ("bwd_dwd_without_gate", "dwd_col[(int64_t)i * hid] += g * elem(dy", "dwd_col[(int64_t)i * hid] += elem(dy"),
    ("bwd_dwg_from_dv", "dwg_row[i] += du * xi;", "dwg_row[i] += dv * xi;"),
    ("bwd_router_dx_dropped", "for (int32_t i = 0; i < d; ++i) dxt[i] += dlt[e]", "for (int32_t i = 0; i < 0; ++i) dxt[i] += dlt[e]"),
    ("bwd_shared_gate_sign", "dls[t] = dsg * sg * (1.0 - sg);", "dls[t] = -dsg * sg * (1.0 - sg);"),
    ("q4_round_down", "float c = rintf(ratio);", "float c = floorf(ratio);"),
    ("q4_scale_over_8", "volatile float s = m / 7.0f;", "volatile float s = m / 8.0f;"),
    ("q4_nibbles_swapped", "(uint8_t)((code[0] + 8) | ((code[1] + 8) << 4))", "(uint8_t)((code[1] + 8) | ((code[0] + 8) << 4))"),
    ("q4_dequant_offset", "out[r * cols + c] = (double)(nib - 8)", "out[r * cols + c] = (double)(nib - 7)"),
    ("bwd_dwr_reversed", "s += dl[t * E + e] * elem(x, t * d + i, c->dtype);",
     "s += dl[t * E + e] * elem(x, t * d + (d - 1 - i), c->dtype);"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, orig, bad):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not found exactly once"
    msrc = tmp_path / "moe_oracle_mutant.c"
    msrc.write_text(src.replace(orig, bad))
    so = str(tmp_path / f"liboracle_{name}.so")
    oracle.build(force=True, source=str(msrc), output=so)
    old = pins.LIB_PATH
    pins.LIB_PATH = so
    failed = []
    try:
        for check in pins.PIN_CHECKS:
            try:
                check()
            except (AssertionError, ValueError, IndexError):
                failed.append(check.__name__)
    finally:
        pins.LIB_PATH = old
        oracle._lib_cache.pop(so, None)
    assert failed, f"planted mistake '{name}' passed every pin"


def test_unmutated_copy_passes(tmp_path):
    so = str(tmp_path / "liboracle_copy.so")
    shutil.copy(SRC, tmp_path / "copy.c")
    oracle.build(force=True, source=str(tmp_path / "copy.c"), output=so)
    old = pins.LIB_PATH
    pins.LIB_PATH = so
    try:
        for check in pins.PIN_CHECKS:
            check()
    finally:
        pins.LIB_PATH = old
