"""Planted mistakes in copies of the oracle must each fail at least one pin.

Every case compiles a copy of oracle/attn_oracle.c with one plausible slip (a dropped term, a
wrong sign, a wrong index, an off-by-one, a transposed operand) into a temporary library and
runs the whole pin suite against it on the CPU. The built oracle itself is never modified.
Every slip keeps the oracle's memory accesses inside its buffers, so a mutant fails by value,
never by corrupting the test process.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

# (name, original text, replacement, which occurrence)
MUTANTS = [
    ("dropped_scale", "s[j] = scale * acc;", "s[j] = acc;", 0),
    ("gqa_index_modulo", "h / group, nk, Nq, Nkv, Sq, Skv, D,\n                 scale, s, out + oo",
     "h % Nkv, nk, Nq, Nkv, Sq, Skv, D,\n                 scale, s, out + oo", 0),
    ("keys_from_next_sequence", "seq_range(layout, cu_kv, b, Skv, &tk0, &lk);",
     "seq_range(layout, cu_kv, (b + 1) % B, Skv, &tk0, &lk);", 0),
    ("values_use_key_head_of_query", "ld(v, offs(layout, b, tk0, j, g, d", "ld(v, offs(layout, b, tk0, j, h % Nkv, d", 0),
    ("causal_off_by_one", "return last + 1 < sk ? last + 1 : sk;", "return last < sk ? last : sk;", 0),
    ("bottomright_sign", "i + sk - sq", "i + sq - sk", 0),
    ("max_not_subtracted", "s[j] = exp(s[j] - mx);", "s[j] = exp(s[j]);", 0),
    ("dropped_normalisation", "for (d = 0; d < D; ++d) o[d] /= sum;\n  *m = mx;",
     "for (d = 0; d < D; ++d) o[d] /= 1.0;\n  *m = mx;", 0),
    ("sequence_search_off_by_one", "while (cu_q[b] <= tok) ++b; /* sequence", "while (cu_q[b] < tok) ++b; /* sequence", 0),
    ("stats_head_major", "(tq0 + i) * Nq + h;", "(tq0 + i) + h * Sq;", 0),
    ("csr_scale_without_sqrt", "1.0 / sqrt((double)D)", "1.0 / (double)D", 0),
    ("csr_first_slice_only", "base = bhi * (int64_t)S * D;", "base = 0;", 0),
    ("csr_query_transposed", "ld(q, rowq + d, et) * ld(k, base + j * D + d, et)",
     "ld(q, base + j * D + d, et) * ld(k, rowq + d, et)", 0),
    ("csr_repeats_counted_once", "s[c - c0] = exp(s[c - c0] - mx);",
     "{ int64_t cc; int seen = 0; for (cc = c0; cc < c; ++cc) seen |= cp[cc] == cp[c];"
     " s[c - c0] = seen ? 0.0 : exp(s[c - c0] - mx); }", 0),
    ("csr_normalisation_dropped", "for (d = 0; d < D; ++d) o[d] /= sum;\n    }\n    free(s);",
     "for (d = 0; d < D; ++d) o[d] /= 1.0;\n    }\n    free(s);", 0),
    ("merge_exp_sign", "prev_sum[x] * exp(pm - m)", "prev_sum[x] * exp(m - pm)", 0),
    ("merge_uses_lane_1", "po = l[0] != 0.0 ? ps_scaled[0] / l[0] : 0.0;",
     "po = l[1] != 0.0 ? ps_scaled[1] / l[1] : 0.0;", 0),
    ("merge_bsh_indexing", "obase = ((s * B + b) * N + n) * (int64_t)D;", "obase = ((b * S + s) * N + n) * (int64_t)D;", 0),
    ("merge_tnd_head_major", "obase = row * (int64_t)D;", "obase = ((row % N) * S + row / N) * (int64_t)D;", 0),
    ("merge_swapped_sides", "ld(prev_out, x, et) * po + ld(cur_out, x, et) * co",
     "ld(prev_out, x, et) * co + ld(cur_out, x, et) * po", 0),
    ("merge_sum_not_rescaled", "cs_scaled[lane] = cur_sum[x] * exp(cm - m);", "cs_scaled[lane] = cur_sum[x];", 0),
    ("cu_order_unchecked", "    if (cu[b] < prev) return -2;\n", "", 0),
    ("cu_total_unchecked", "  if (B > 0 && prev != T) return -2;\n", "", 0),
    ("csr_rowptr_start_unchecked", "if (op[0] != 0 || op[S] > nnz_cap) return -2;", "if (op[S] > nnz_cap) return -2;", 0),
    ("csr_rowptr_order_unchecked", "      if (op[r + 1] < op[r]) return -2;\n", "", 0),
    ("bf16_decode_unshifted", "uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;",
     "uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]);", 0),
    ("bf16_truncates", "nearbyint(m * 256.0)", "floor(m * 256.0)", 0),
    ("f16_truncates", "nearbyint(m * 2048.0)", "floor(m * 2048.0)", 0),
    ("f16_subnormal_grid_off", "nearbyint(a * 0x1p24)", "nearbyint(a * 0x1p23) * 2.0", 0),
    ("f16_exponent_bias_off", "(e - 1 + 15) << 10", "(e + 15) << 10", 0),
    ("band_lower_off_by_one", "(j < i - pre || j > i + next)", "(j <= i - pre || j > i + next)", 0),
    ("band_upper_sign", "(j < i - pre || j > i + next)", "(j < i - pre || j > i - next)", 0),
    ("mask_polarity", "mask[mrow + i * mask_rstride + j] != 0", "mask[mrow + i * mask_rstride + j] == 0", 0),
    ("mask_row_stride_ignored", "mask[mrow + i * mask_rstride + j]", "mask[mrow + i * sk + j]", 0),
    ("mask_batch_stride_ignored", "b * mask_bstride, mask_rstride))", "0 * mask_bstride, mask_rstride))", 0),
    ("mask_key_shifted", "mask[mrow + i * mask_rstride + j]", "mask[mrow + i * mask_rstride + (j + 1) % sk]", 0),
    ("ext_dropped_scale", "s[j] = scale * acc;", "s[j] = acc;", 1),
    ("ext_max_not_subtracted", "s[j] == -INFINITY ? 0.0 : exp(s[j] - mx);", "s[j] == -INFINITY ? 0.0 : exp(s[j]);", 0),
    ("ext_normalisation_dropped", "for (d = 0; d < Dv; ++d) o[d] /= sum;", "for (d = 0; d < Dv; ++d) o[d] /= 1.0;", 0),
    ("empty_row_max_zero", "    *m = -INFINITY;\n    *l = 0.0;\n    return;", "    *m = 0.0;\n    *l = 0.0;\n    return;", 0),
    ("ext_empty_row_max_zero", "    *m = -INFINITY;\n    *l = 0.0;\n    return;", "    *m = 0.0;\n    *l = 0.0;\n    return;", 1),
    ("merge_max_is_min", "double m = pm > cm ? pm : cm;", "double m = pm < cm ? pm : cm;", 0),
    ("ext_gqa_next_head", "h / group, lq, lk,", "(h / group + 1) % Nkv, lq, lk,", 0),
    ("mask_replaces_mode", "  if (mask_mode == ORC_MASK_TOPLEFT && j > i) return 0;",
     "  if (mask != NULL) return mask[mrow + i * mask_rstride + j] == 0;\n"
     "  if (mask_mode == ORC_MASK_TOPLEFT && j > i) return 0;", 0),
    ("band_bottom_right_aligned", "(j < i - pre || j > i + next)",
     "(j < i + sk - sq - pre || j > i + sk - sq + next)", 0),
    ("csr_empty_row_divides", "      if (c1 <= c0) continue;\n", "", 0),
    ("merge_stats_sum_from_lane_0", "out_sum[x] = l[lane];", "out_sum[x] = l[0];", 0),
    ("merge_cur_scaled_by_prev_max", "cs_scaled[lane] = cur_sum[x] * exp(cm - m);",
     "cs_scaled[lane] = cur_sum[x] * exp(pm - m);", 0),
    ("scores_over_value_dims", "for (d = 0; d < Dqk; ++d)\n      acc +=", "for (d = 0; d < Dv; ++d)\n      acc +=", 0),
]


def _mutate(text, old, new, nth):
    pos = -1
    for _ in range(nth + 1):
        pos = text.find(old, pos + 1)
        assert pos >= 0, f"mutation anchor not found: {old!r}"
    return text[:pos] + new + text[pos + len(old):]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant's NaN or inf in the pins' arithmetic
@pytest.mark.parametrize("name,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, nth, tmp_path):
    src = open(SRC).read()
    mutated = _mutate(src, old, new, nth)
    assert mutated != src
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"],
                   check=True)
    failed = []
    with oracle.using(str(so)):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except Exception:  # an assertion, or the mutant rejecting valid input
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
