"""GPU parity of the router's fp32 logits (gqe_route_train) and of the
load-balancing auxiliary loss (gqe_aux_loss) against the CPU oracle.

Tolerances: logits within 1e-4 of the oracle's (fp32 sums of up to 4096 bf16
products of unit scale, accumulated in different orders); the loss within 1e-5
relative; the logit gradient c * p * (f_j - sum_i p_i f_i), c = (h/g)/(g N),
within 1e-6 * c: its terms are of size c at most, and near-uniform routing makes
their difference (the gradient itself) much smaller, so fp32 rounding is
measured against the terms, not against the result."""
import numpy as np
import pytest
import torch

import gqe_synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

W = gqe_synth.WORKLOADS
C = gqe_synth.custom

CASES = [
    C("aux_k1", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=1, seed=91),
    C("aux_k2_skew", B=1, T=520, d_model=96, h=16, g=8, d_h=128, k=1, head0_bias=1.0, seed=92),
    C("aux_h64_k3", B=2, T=96, d_model=256, h=64, g=8, d_h=128, k=3, seed=93),
    C("aux_f32", B=2, T=100, d_model=48, h=8, g=2, d_h=64, k=2, dtype="f32", seed=94),
    W["gqe_prefill"],
    W["gqe_long"],
]


def _aux_on_gpu(g, w, logits, idx):
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    ws = torch.zeros(g.gqe_aux_loss_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    loss = torch.full((1,), float("nan"), device="cuda")
    dl = torch.full((w.B * w.T, w.h), float("nan"), device="cuda")
    g.gqe_aux_loss(shape, logits, idx, loss, dl, ws)
    torch.cuda.synchronize()
    st = g.gqe_get_device_status(ws)
    assert st == 0, g.gqe_status_string(st)
    return float(loss.item()), dl.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_route_logits_and_aux_loss(w):
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, "cuda")
    logits = torch.full((w.B * w.T, w.h), float("nan"), device="cuda")
    g.gqe_route_train(shape, U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]), buf.idx, buf.gate,
                      buf.head_offsets, buf.head_pos, buf.head_chunk_offsets, logits, buf.workspace)
    torch.cuda.synchronize()
    assert buf.status() == 0
    idx_o, gate_o, logits_o, margin_o = U.oracle_route(w, inp)
    err_l = float(np.abs(logits.cpu().numpy().astype(np.float64) - logits_o.reshape(-1, w.h)).max())
    assert err_l <= 1e-4, f"{w.name}: logits differ by {err_l}"
    excl, _, _ = U.check_routing(w, inp, buf.idx, buf.gate)  # the same selection as gqe_route

    # the loss kernel on the oracle's own logits and selection: a strict comparison
    lo = torch.from_numpy(np.ascontiguousarray(logits_o.reshape(-1, w.h), dtype=np.float32)).cuda()
    io = torch.from_numpy(np.ascontiguousarray(idx_o, dtype=np.int32)).cuda()
    loss_g, dl_g = _aux_on_gpu(g, w, lo, io)
    loss_o, dl_o = oracle.aux_loss(logits_o, idx_o)
    dl_o = dl_o.reshape(-1, w.h)
    assert abs(loss_g - loss_o) <= 1e-5 * abs(loss_o), f"{w.name}: loss {loss_g} vs {loss_o}"
    c = (w.h // w.g) / (w.g * w.B * w.T)
    assert np.abs(dl_g - dl_o).max() <= 1e-6 * c, f"{w.name}: dlogits error {np.abs(dl_g - dl_o).max()} (c = {c})"

    # end to end on the GPU's own logits and selection: equal up to the excluded
    # near-tie tokens (each moves one selection count by 1/(N k))
    loss_e, _ = _aux_on_gpu(g, w, logits, buf.idx)
    n_excl = int(excl.sum())
    bound = 1e-5 * abs(loss_o) + n_excl * w.g * (w.h // w.g) / (w.B * w.T * w.k) * 2.0
    assert abs(loss_e - loss_o) <= bound, f"{w.name}: end-to-end loss {loss_e} vs {loss_o} ({n_excl} excluded)"


def test_aux_loss_balanced_and_repeatable():
    """Equal logits and a selection that gives every head the same count: the
    loss is exactly 1 and the gradient is zero (the reading's balanced case);
    two runs give bit-identical results."""
    g = U.gqe()
    w = C("aux_bal", B=1, T=256, d_model=32, h=8, g=2, d_h=128, k=2, seed=95)
    N, hpg = w.B * w.T, w.h // w.g
    logits = torch.zeros((N, w.h), device="cuda")
    sel = np.zeros((N, w.g, w.k), np.int32)
    for t in range(N):
        for q in range(w.g):
            a = (2 * t) % hpg
            sel[t, q] = [q * hpg + a, q * hpg + (a + 1) % hpg]
    idx = torch.from_numpy(sel).cuda()
    l1, d1 = _aux_on_gpu(g, w, logits, idx)
    l2, d2 = _aux_on_gpu(g, w, logits, idx)
    assert abs(l1 - 1.0) <= 1e-6 and np.abs(d1).max() <= 1e-9
    assert l1 == l2 and np.array_equal(d1, d2)
