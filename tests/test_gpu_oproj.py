"""GPU parity of the routed output projection (gqe_routed_oproj) against the
CPU oracle on the same seeded inputs: each token's output row equals the sum,
over the heads it selected, of O[b,t,j,:] . W_Z[j-block] within the bf16
tolerance (2e-2 max-abs).  The routing is a seeded draw with the router's
structure (k distinct heads per group); O holds N(0, 1/2) in the selected
slots and zeros elsewhere, as the routed prefill writes it."""
import numpy as np
import pytest
import torch

import gqe_synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

C = gqe_synth.custom

SMALL = [
    # ragged B*T (a partial last token tile), d_model not a multiple of 256 (a partial column tile)
    (C("op_k2", B=2, T=300, d_model=288, h=8, g=2, d_h=128, k=2, seed=91), False),
    (C("op_h32_k1", B=1, T=200, d_model=512, h=32, g=8, d_h=128, k=1, seed=92), False),
    (C("op_dense", B=1, T=129, d_model=256, h=8, g=2, d_h=128, k=4, seed=93), False),
    (C("op_dh64", B=3, T=70, d_model=96, h=16, g=8, d_h=64, k=1, seed=94), False),
    (C("op_T1", B=5, T=1, d_model=64, h=8, g=2, d_h=128, k=2, seed=95), False),
    # the first 128 tokens all take each group's first k heads: the other heads
    # are skipped for that tile
    (C("op_skip", B=1, T=384, d_model=512, h=32, g=8, d_h=128, k=2, seed=96), True),
]


def run_oproj(w, first_tile_fixed=False):
    g = U.gqe()
    idx = gqe_synth.make_random_routing(w, first_tile_fixed=first_tile_fixed)
    O = gqe_synth.make_routed_output(w, idx)
    W_Z = gqe_synth.make_oproj_weight(w)
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    ws = torch.zeros(g.gqe_workspace_bytes(shape, 0), dtype=torch.uint8, device="cuda")
    g.gqe_workspace_init(ws)
    Y = torch.full((w.B, w.T, w.d_model), float("nan"), dtype=w.torch_dtype, device="cuda")
    args = (shape, U.to_dev(O), U.to_dev(idx), U.to_dev(W_Z))
    g.gqe_routed_oproj(*args, Y, ws)
    torch.cuda.synchronize()
    assert g.gqe_get_device_status(ws) == 0
    return idx, O, W_Z, Y, args, ws


def compare(w, idx, O, W_Z, Y, rows):
    rows = np.asarray(rows, dtype=np.int64)
    want = oracle.oproj_rows(O, W_Z, idx.numpy(), rows=rows)
    got = Y.float().reshape(w.B * w.T, w.d_model)[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), "unwritten output element"
    return float(np.abs(got - want).max(initial=0.0))


@pytest.mark.parametrize("w,fixed", SMALL, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_oproj_small(w, fixed):
    idx, O, W_Z, Y, _, _ = run_oproj(w, fixed)
    err = compare(w, idx, O, W_Z, Y, np.arange(w.B * w.T))
    assert err <= U.TOL["bf16"], f"{w.name}: max |Y - oracle| = {err}"


def test_oproj_full_size_sampled_and_repeatable():
    """gqe_prefill shapes (B=8, T=4096, h=32, g=8, k=2, d_model=4096): three whole
    128-token tiles (the first, one in the middle, the last) and the last
    position of every sequence against the oracle, and a second call
    bit-identical to the first."""
    w = gqe_synth.WORKLOADS["gqe_prefill"]
    idx, O, W_Z, Y, args, ws = run_oproj(w)
    BT = w.B * w.T
    mid = (BT // 128 // 2) * 128
    rows = np.unique(np.concatenate([np.arange(128), np.arange(mid, mid + 128), np.arange(BT - 128, BT),
                                     np.arange(1, w.B + 1) * w.T - 1]))
    err = compare(w, idx, O, W_Z, Y, rows)
    assert err <= U.TOL["bf16"], f"full size: max |Y - oracle| = {err} over {len(rows)} rows"
    U.gqe().gqe_routed_oproj(*args, Y2 := torch.empty_like(Y), ws)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2), "two calls differ"


def test_oproj_reports_foreign_index():
    """A head index outside [0, h) is reported in the status word; the call
    still completes and the other rows are right."""
    g = U.gqe()
    w = SMALL[0][0]
    idx = gqe_synth.make_random_routing(w)
    O = gqe_synth.make_routed_output(w, idx)
    W_Z = gqe_synth.make_oproj_weight(w)
    bad = idx.clone()
    bad[0, 3, 0, 0] = w.h + 5
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    ws = torch.zeros(g.gqe_workspace_bytes(shape, 0), dtype=torch.uint8, device="cuda")
    g.gqe_workspace_init(ws)
    Y = torch.empty((w.B, w.T, w.d_model), dtype=w.torch_dtype, device="cuda")
    g.gqe_routed_oproj(shape, U.to_dev(O), U.to_dev(bad), U.to_dev(W_Z), Y, ws)
    torch.cuda.synchronize()
    assert g.gqe_get_device_status(ws) == g.GQE_ERR_INVALID_ARGUMENT
    rows = np.arange(128, w.B * w.T)  # the token tiles without the bad index
    assert compare(w, idx, O, W_Z, Y, rows) <= U.TOL["bf16"]
