"""The pins have teeth: each plausible mistake, planted in a copy of the
oracle's C source on the CPU, makes at least one pin in oracle_pins.py fail.

Each mutant is compiled into a temporary library and checked in a child
process (a broken copy may crash)."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

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
    ("topk_picks_smallest", "if (lg[prev] < lg[a]) {", "if (lg[prev] > lg[a]) {"),
    ("margin_from_top_logit", "(double)lg[order[k - 1]] - (double)lg[order[k]]", "(double)lg[order[0]] - (double)lg[order[k]]"),
    ("compact_first_slot_only", "for (int s = 0; s < k; ++s) hit |= (sel[s] == j);",
     "for (int s = 0; s < 1; ++s) hit |= (sel[s] == j);"),
    ("compact_drops_last_position", "for (int t = 0; t < T; ++t) {\n                const int32_t* sel",
     "for (int t = 0; t < T - 1; ++t) {\n                const int32_t* sel"),
    ("slots_query_from_slot_not_head", "attend_one(Q, ((size_t)bt * h + j) * d_h, K, V",
     "attend_one(Q, ((size_t)bt * h + q * hpg + s) * d_h, K, V"),
    ("weighted_sum_first_gate", "for (int d = 0; d < d_h; ++d) ws[d] += gate[sel] * slot[d];",
     "for (int d = 0; d < d_h; ++d) ws[d] += gate[sel - s] * slot[d];"),
    ("oproj_reads_slot_not_head", "load_elem(O, ((size_t)bt * h + jh) * d_h + c, dtype)",
     "load_elem(O, ((size_t)bt * h + q * (h / g) + s) * d_h + c, dtype)"),
    ("paged_scale_dropped", "load_elem(K_pages, row + d, dtype);\n                            scores[s] = dot * scale;",
     "load_elem(K_pages, row + d, dtype);\n                            scores[s] = dot;"),
    ("paged_gate_dropped", "const double w = gate[sel] * scores[s] / denom;", "const double w = scores[s] / denom;"),
    ("paged_query_from_slot", "const size_t q_off = ((size_t)b * h + j) * d_h;\n                        /* scores",
     "const size_t q_off = ((size_t)b * h + q * hpg + r) * d_h;\n                        /* scores"),
    ("bwd_query_from_slot", "const size_t q_off = (((size_t)b * T + t) * h + j) * d_h;",
     "const size_t q_off = (((size_t)b * T + t) * h + q * hpg + s_) * d_h;"),
    ("bwd_dgate_gated", "for (int d = 0; d < d_h; ++d) dg += dO[q_off + d] * o[d];",
     "for (int d = 0; d < d_h; ++d) dg += gate[sel] * dO[q_off + d] * o[d];"),
    ("bwd_weights_unnormalised", "for (int s = 0; s <= t; ++s) p[s] /= denom;", "for (int s = 0; s <= t; ++s) p[s] /= 1.0;"),
    ("router_bwd_dlogits_slot_head", "dlogits[bt * h + idx[base + s]] = gate",
     "dlogits[bt * h + q * hpg + s] = gate"),
    ("slots_in_reverse_order", "double* slot = cat_rows + (((size_t)r * g + q) * k + s) * d_h;",
     "double* slot = cat_rows + (((size_t)r * g + q) * k + (k - 1 - s)) * d_h;"),
]

_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins
oracle.compile_source({src!r}, {lib!r}, strict=False)
o = oracle.Oracle({lib!r})
failed = []
for c in oracle_pins.ALL_CHECKS:
    try:
        c(o)
    except Exception as e:
        failed.append(c.__name__)
print("FAILED:" + ",".join(failed))
"""


def _check_mutant(tmp_dir, name, old, new):
    """Plant one mistake (at the anchor's first occurrence) in a copy of the
    oracle's source, build it and run every pin against it in a child
    process.  Returns (anchor found, caught, child output)."""
    src = open(oracle.SOURCE).read()
    if src.count(old) < 1:
        return False, False, ""
    c_path = os.path.join(tmp_dir, name + ".c")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new, 1))
    lib = os.path.join(tmp_dir, "lib" + name + ".so")
    env = dict(os.environ, OMP_NUM_THREADS="1", OMP_WAIT_POLICY="PASSIVE")
    proc = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, src=c_path, lib=lib)],
                          capture_output=True, text=True, timeout=600, env=env)
    caught = proc.returncode != 0 or ("FAILED:" in proc.stdout and proc.stdout.split("FAILED:")[1].strip() != "")
    return True, caught, proc.stdout + proc.stderr[-2000:]


@pytest.fixture(scope="module")
def verdicts(tmp_path_factory):
    """Every mutant checked once, in child processes run side by side (each
    child spends most of its time importing torch)."""
    tmp_dir = str(tmp_path_factory.mktemp("mutants"))
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {m[0]: ex.submit(_check_mutant, tmp_dir, *m) for m in MUTANTS}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_mutant_is_caught(verdicts, name):
    found, caught, out = verdicts[name]
    assert found, f"mutation anchor of {name} not found in the oracle's source"
    assert caught, f"mutant {name} passed every pin:\n{out}"
