"""GPU parity of the routed query projection (gqe_routed_qproj) against the
CPU oracle on the same seeded inputs: every routed (t, j) row of Q equals
x[b,t] . W_Q[:, j-block] within the bf16 tolerance (2e-2 max-abs); rows of
unselected heads are left untouched."""
import numpy as np
import pytest
import torch

import gqe_synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

W = gqe_synth.WORKLOADS
C = gqe_synth.custom

SMALL = [
    C("qp_k2", B=2, T=300, d_model=256, h=8, g=2, d_h=128, k=2, seed=81),
    C("qp_h32_k1", B=1, T=200, d_model=512, h=32, g=8, d_h=128, k=1, seed=82),
    C("qp_dense_k4", B=1, T=129, d_model=128, h=8, g=2, d_h=128, k=4, seed=83),
    C("qp_T1", B=3, T=1, d_model=64, h=8, g=2, d_h=128, k=2, seed=84),
    C("qp_skew_d96", B=1, T=150, d_model=96, h=16, g=8, d_h=128, k=1, head0_bias=1.0, seed=85),
]

SENTINEL = -12288.0  # -1.5 * 2^13: exactly representable in bf16


def qproj_parity(w, rows=None, cover=False, gather=False):
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    W_Q = gqe_synth.make_qproj_weight(w)
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, "cuda")
    buf.route(U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]))
    Qp = torch.full((w.B, w.T, w.h, w.d_h), SENTINEL, dtype=w.torch_dtype, device="cuda")
    ws = buf.workspace if not gather else buf.workspace[: 256]  # a status-word-only workspace: the gather path
    g.gqe_routed_qproj(shape, U.to_dev(inp["x"]), U.to_dev(W_Q), buf.idx, buf.head_offsets, buf.head_pos, Qp, ws)
    torch.cuda.synchronize()
    assert buf.status() == 0
    excl, idx_o, _ = U.check_routing(w, inp, buf.idx, buf.gate)
    if cover:
        rows = U.cover_rows(w, idx_o, U.sm_count())
    if rows is None:
        rows = np.arange(w.B * w.T)
    rows = np.asarray(rows, dtype=np.int64)
    rows = rows[~excl.reshape(-1)[rows]]
    want = oracle.qproj_rows(inp["x"], W_Q, idx_o, w.d_h, rows=rows)  # [n, g, k, d_h]
    got_all = Qp.float().reshape(w.B * w.T, w.h, w.d_h)[torch.from_numpy(rows).cuda()].cpu().numpy()
    sel = idx_o.reshape(w.B * w.T, w.g * w.k)[rows]  # [n, g*k]
    got = np.take_along_axis(got_all, sel[:, :, None].astype(np.int64), axis=1).reshape(want.shape)
    err = float(np.abs(got.astype(np.float64) - want).max(initial=0.0))
    # rows of unselected heads keep the sentinel
    mask = np.ones((len(rows), w.h), bool)
    np.put_along_axis(mask, sel.astype(np.int64), False, axis=1)
    untouched = bool((got_all[mask] == SENTINEL).all())
    return err, len(rows), untouched


@pytest.mark.parametrize("gather", [False, True], ids=["auto", "gather"])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_qproj_small(w, gather):
    """auto: the dense tiled path where the routed share g*k/h >= 3/10 (all but
    qp_h32_k1), else the gathered rows; gather: a status-word-only workspace
    forces the gathered path."""
    err, n, untouched = qproj_parity(w, gather=gather)
    assert n > 0
    assert err <= U.TOL["bf16"], f"{w.name}: max abs error {err} over {n} rows"
    assert untouched, "rows of unselected heads were written"


@pytest.mark.parametrize("name,gather", [("dense_gqa", False), ("gqe_prefill", False), ("gqe_long", False),
                                         ("gqe_prefill", True)])
def test_qproj_full_size_covered(name, gather):
    """At least 4096 token rows (every routed head of each): whole windows of
    consecutive positions (first, middle and last prefill units of three CTAs,
    each sequence's last window, the most skewed windows) plus random rows; the
    gathered path once at full size as well."""
    w = W[name]
    err, n, untouched = qproj_parity(w, cover=True, gather=gather)
    assert n >= 4096 - 64, f"{name}: only {n} rows compared"
    assert err <= U.TOL["bf16"], f"{name}: max abs error {err} over {n} rows"
    assert untouched
