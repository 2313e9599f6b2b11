"""The pins have teeth: each plausible mistake, planted in a copy of the
oracle's C source on the CPU, makes at least one pin in oracle_pins.py fail.

Each mutant is compiled into a temporary library and checked in a child
process (a broken copy may crash)."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, original text, planted mistake)
MUTANTS = [
    ("scale_1_over_d", "1.0 / sqrt((double)d_h)", "1.0 / (double)d_h"),
    ("causal_excludes_diagonal", "t + 1, d_h, dtype,", "t, d_h, dtype,"),
    ("causal_sees_one_future_key", "t + 1, d_h, dtype,", "(t + 1 < T ? t + 2 : t + 1), d_h, dtype,"),
    ("strided_head_group_map", "idx[o] = q * hpg + order[s];", "idx[o] = order[s] * g + q;"),
    ("ties_to_higher_index", "if (lg[prev] < lg[a]) {", "if (lg[prev] <= lg[a]) {"),
    ("gate_over_all_group_heads", "for (int s = 0; s < k; ++s) denom +=", "for (int s = 0; s < hpg; ++s) denom +="),
    ("transposed_router_weight", "load_elem(W_r, (size_t)i * h + j, dtype)", "load_elem(W_r, ((size_t)j * d_model + i) % ((size_t)d_model * h), dtype)"),
    ("dropped_bias", "if (bias) acc += (double)bias[j];", "(void)bias;"),
    ("unnormalised_weights", "const double w = scores[s] / denom;", "const double w = scores[s];"),
    ("decode_query_position", "lengths[b], d_h, dtype, scores, o);", "lengths[b] - 1 > 0 ? lengths[b] - 1 : 1, d_h, dtype, scores, o);"),
    ("gate_not_applied", "out[(size_t)j * d_h + d] = gate[sel] * o[d];", "out[(size_t)j * d_h + d] = o[d];"),
    ("unselected_heads_not_zero", "for (int i = 0; i < h * d_h; ++i) out[i] = 0.0;", "for (int i = 0; i < h * d_h; ++i) out[i] = 1e-3;"),
    ("transposed_qk_index", "load_elem(K, kr + d, dtype)", "load_elem(K, kv_base + (size_t)d * kv_row_stride + (size_t)s % (size_t)d_h, dtype)"),
    ("compact_strided_group", "const int q = j / hpg;", "const int q = j % g;"),
    ("shared_head_group_0", "const size_t kv_base = ((size_t)b * T * g + kv_group) * d_h;",
     "const size_t kv_base = ((size_t)b * T * g + 0) * d_h;"),
    ("shared_head_sees_all_keys", "(size_t)g * d_h, t + 1, d_h, dtype,\n                           scores, Os_rows",
     "(size_t)g * d_h, T, d_h, dtype,\n                           scores, Os_rows"),
    ("weighted_sum_ungated", "for (int d = 0; d < d_h; ++d) ws[d] += gate[sel] * slot[d];",
     "for (int d = 0; d < d_h; ++d) ws[d] += slot[d];"),
    ("qproj_head_block_offset", "load_elem(W_Q, (size_t)i * ldw + (size_t)j * d_h + c, dtype);",
     "load_elem(W_Q, (size_t)i * ldw + (size_t)j + c, dtype);"),
    ("qproj_transposed_weight", "load_elem(W_Q, (size_t)i * ldw + (size_t)j * d_h + c, dtype);",
     "load_elem(W_Q, ((size_t)((size_t)j * d_h + c) * d_model + i) % ((size_t)d_model * ldw), dtype);"),
    ("oproj_head_block_offset", "load_elem(W_Z, ((size_t)jh * d_h + c) * d_model + n, dtype);",
     "load_elem(W_Z, ((size_t)jh + c) * d_model + n, dtype);"),
    ("oproj_transposed_weight", "load_elem(W_Z, ((size_t)jh * d_h + c) * d_model + n, dtype);",
     "load_elem(W_Z, ((size_t)n * h * d_h + (size_t)jh * d_h + c) % ((size_t)h * d_h * d_model), dtype);"),
    ("oproj_unrouted_heads", "const int jh = idx[((size_t)bt * g + q) * k + s];",
     "const int jh = q * (h / g) + s;"),
    ("paged_row_offset", "const size_t row = ((pg * page_size + (size_t)(s % page_size)) * g + q) * d_h;",
     "const size_t row = ((pg * page_size + (size_t)((s + 1) % page_size)) * g + q) * d_h;"),
    ("paged_block_lookup", "(size_t)block_table[(size_t)b * max_blocks + s / page_size];",
     "(size_t)block_table[(size_t)b * max_blocks + (s / page_size) % 2];"),
    ("bwd_drops_softmax_mean", "const double dz = p[s] * (dp[s] - pdp);", "const double dz = p[s] * dp[s];"),
    ("bwd_output_grad_ungated", "dov[d] = gate[sel] * dO[q_off + d];", "dov[d] = dO[q_off + d];"),
    ("bwd_dk_from_key", "dK[kr + d] += scale * dz * load_elem(Q, q_off + d, dtype);",
     "dK[kr + d] += scale * dz * load_elem(K, kr + d, dtype);"),
    ("bwd_dq_unscaled", "dQ[q_off + d] += scale * dz * load_elem(K, kr + d, dtype);",
     "dQ[q_off + d] += dz * load_elem(K, kr + d, dtype);"),
    ("bwd_dv_uniform_weights", "dV[kr + d] += p[s] * dov[d];", "dV[kr + d] += dov[d] / (double)(t + 1);"),
    ("router_bwd_drops_mean", "gate[base + s] * (dgate[base + s] - mean);", "gate[base + s] * dgate[base + s];"),
    ("router_bwd_dx_transposed", "acc += dlogits[bt * h + j] * load_elem(W_r, (size_t)i * h + j, dtype);",
     "acc += dlogits[bt * h + j] * load_elem(W_r, ((size_t)j * d_model + i) % ((size_t)d_model * h), dtype);"),
    ("router_bwd_dw_wrong_head", "acc += load_elem(x, (size_t)bt * d_model + i, dtype) * dlogits[bt * h + j];",
     "acc += load_elem(x, (size_t)bt * d_model + i, dtype) * dlogits[bt * h + (j + 1) % h];"),
    ("router_bwd_dbias_halved", "dbias[j] = acc;", "dbias[j] = 0.5 * acc;"),
    ("aux_fraction_per_token", "f[j] += 1.0 / ((double)N * k);", "f[j] += 1.0 / (double)N;"),
    ("aux_no_group_size_factor", "L += (double)hpg * s / (double)g;", "L += s / (double)g;"),
    ("aux_grad_drops_mean", "c * p[jj] * (f[q * hpg + jj] - pf);", "c * p[jj] * f[q * hpg + jj];"),
    ("query_row_from_slot_not_head", "const size_t q_off = ((size_t)bt * h + j) * d_h;",
     "const size_t q_off = ((size_t)bt * h + q * hpg + s) * d_h;"),
    ("kv_group_strided", "const size_t kv_base = ((size_t)b * T * g + q) * d_h;",
     "const size_t kv_base = ((size_t)b * T * g + j % g) * d_h;"),
    ("values_read_from_keys", "o[d] += w * load_elem(V, vr + d, dtype);", "o[d] += w * load_elem(K, vr + d, dtype);"),
    ("decode_output_in_slot_order", "O[((size_t)b * h + j) * d_h + d] = gate[sel] * o[d];",
     "O[((size_t)b * h + q * hpg + s) * d_h + d] = gate[sel] * o[d];"),
    ("decode_kv_group_strided", "const size_t kv_base = ((size_t)b * Lmax * g + q) * d_h;",
     "const size_t kv_base = ((size_t)b * Lmax * g + j % g) * d_h;"),
    ("slots_in_reverse_order", "double* slot = cat_rows + (((size_t)r * g + q) * k + s) * d_h;",
     "double* slot = cat_rows + (((size_t)r * g + q) * k + (k - 1 - s)) * d_h;"),
]

_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins
o = oracle.Oracle({lib!r})
failed = []
for c in oracle_pins.ALL_CHECKS:
    try:
        c(o)
    except Exception as e:
        failed.append(c.__name__)
print("FAILED:" + ",".join(failed))
"""


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new, 1)  # one planted mistake, at the anchor's first occurrence
    c_path = tmp_path / "mutant.c"
    c_path.write_text(mutated)
    lib = str(tmp_path / "libmutant.so")
    oracle.compile_source(str(c_path), lib, strict=False)
    proc = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, lib=lib)],
                          capture_output=True, text=True, timeout=300)
    caught = proc.returncode != 0 or ("FAILED:" in proc.stdout and proc.stdout.split("FAILED:")[1].strip())
    assert caught, f"mutant {name} passed every pin:\n{proc.stdout}\n{proc.stderr[-2000:]}"
