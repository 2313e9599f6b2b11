"""GPU parity of the GQE output construction: the always-active shared head
and the per-group slots (concatenated expert outputs, gate-weighted sum),
through the C ABI, against the CPU oracle on the same seeded inputs.
Tolerances as for the routed heads: max-abs 1e-4 (fp32), 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import gqe_synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

W = gqe_synth.WORKLOADS
C = gqe_synth.custom

SHARED = [
    (C("sh_bf16", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=1, seed=61), 1),
    (C("sh_bf16_T129_g4", B=1, T=129, d_model=64, h=8, g=4, d_h=128, k=1, seed=62), 3),
    (C("sh_bf16_T1", B=3, T=1, d_model=64, h=8, g=2, d_h=128, k=1, seed=63), 0),
    (C("sh_f32_d64", B=2, T=100, d_model=32, h=4, g=2, d_h=64, k=1, dtype="f32", seed=64), 1),
]


def run_shared(w, kv_group):
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    Qs = gqe_synth.make_shared_query(w)
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    ws = torch.empty(g.gqe_workspace_bytes(shape, 0), dtype=torch.uint8, device="cuda")
    g.gqe_workspace_init(ws)
    Os = torch.empty((w.B, w.T, w.d_h), dtype=w.torch_dtype, device="cuda")
    g.gqe_attn_shared_head(shape, U.to_dev(Qs), U.to_dev(inp["K"]), U.to_dev(inp["V"]), kv_group, Os, ws)
    torch.cuda.synchronize()
    st = g.gqe_get_device_status(ws)
    assert st == 0, g.gqe_status_string(st)
    return inp, Qs, Os


@pytest.mark.parametrize("w,kv", SHARED, ids=[c[0].name for c in SHARED])
def test_shared_head_small(w, kv):
    inp, Qs, Os = run_shared(w, kv)
    want = oracle.shared_rows(Qs, inp["K"], inp["V"], kv).reshape(w.B, w.T, w.d_h)
    err = float(np.abs(Os.float().cpu().numpy().astype(np.float64) - want).max())
    assert err <= U.TOL[w.dtype], f"{w.name}: shared head max abs error {err}"


def test_shared_head_full_size_sampled():
    """The dense_gqa shapes in the bench's launch configuration (KV group 5),
    on 4096 sampled rows (each sequence's last position included)."""
    w, kv = W["dense_gqa"], 5
    inp, Qs, Os = run_shared(w, kv)
    rows = gqe_synth.sample_rows(w, 4096).numpy()
    want = oracle.shared_rows(Qs, inp["K"], inp["V"], kv, rows=rows)
    got = Os.float().reshape(w.B * w.T, w.d_h)[torch.from_numpy(rows).cuda()].cpu().numpy()
    err = float(np.abs(got.astype(np.float64) - want).max())
    assert err <= U.TOL["bf16"], f"shared head max abs error {err}"


SLOTS = [
    C("sl_bf16_k2", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=2, seed=71),
    C("sl_bf16_k4_dense", B=1, T=257, d_model=64, h=8, g=2, d_h=128, k=4, seed=72),
    C("sl_bf16_k1", B=1, T=200, d_model=96, h=16, g=8, d_h=128, k=1, head0_bias=1.0, seed=73),
    C("sl_f32_k2", B=2, T=100, d_model=48, h=8, g=2, d_h=64, k=2, dtype="f32", seed=74),
]


def slots_parity(w, rows=None, cover=False):
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    buf = U.run_prefill(w, inp)
    excl, idx_o, gate_o = U.check_routing(w, inp, buf.idx, buf.gate)
    # the slot order follows the selection order: also skip tokens whose order
    # is a near-tie on the oracle's own logits
    _, _, logits_o, _ = U.oracle_route(w, inp)
    lg_sel = np.take_along_axis(logits_o.astype(np.float64)[:, :, None, :].repeat(w.g, 2), idx_o, axis=-1)
    if w.k > 1:
        excl = excl | (np.abs(lg_sel[..., :-1] - lg_sel[..., 1:]) < U.MARGIN_EXCLUDE).any(axis=(-1, -2))
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    cat = torch.empty((w.B, w.T, w.g, w.k, w.d_h), dtype=w.torch_dtype, device="cuda")
    wsum = torch.empty((w.B, w.T, w.g, w.d_h), dtype=w.torch_dtype, device="cuda")
    g.gqe_group_slots(shape, buf.O, buf.idx, buf.gate, cat, wsum)
    torch.cuda.synchronize()
    if cover:
        rows = U.cover_rows(w, idx_o, U.sm_count())
    if rows is None:
        rows = np.arange(w.B * w.T)
    rows = np.asarray(rows, dtype=np.int64)
    rows = rows[~excl.reshape(-1)[rows]]
    want_c, want_w = oracle.group_slots_rows(inp["Q"], inp["K"], inp["V"], idx_o, gate_o, rows=rows)
    sel = torch.from_numpy(rows).cuda()
    got_c = cat.float().reshape(w.B * w.T, w.g, w.k, w.d_h)[sel].cpu().numpy().astype(np.float64)
    got_w = wsum.float().reshape(w.B * w.T, w.g, w.d_h)[sel].cpu().numpy().astype(np.float64)
    return float(np.abs(got_c - want_c).max(initial=0.0)), float(np.abs(got_w - want_w).max(initial=0.0)), len(rows)


@pytest.mark.parametrize("w", SLOTS, ids=lambda w: w.name)
def test_group_slots_small(w):
    ec, ew, n = slots_parity(w)
    assert n > 0
    assert ec <= U.TOL[w.dtype] and ew <= U.TOL[w.dtype], f"{w.name}: cat {ec}, wsum {ew} over {n} rows"


@pytest.mark.parametrize("name", ["dense_gqa", "gqe_prefill"])
def test_group_slots_full_size_covered(name):
    """At least 4096 rows: whole prefill work units of a first, a middle and the
    last CTA, every sequence's last window, the most skewed windows, random rows."""
    w = W[name]
    ec, ew, n = slots_parity(w, cover=True)
    assert n >= 4096 - 64, f"{name}: only {n} rows compared"
    assert ec <= U.TOL["bf16"] and ew <= U.TOL["bf16"], f"{name}: cat {ec}, wsum {ew} over {n} rows"
