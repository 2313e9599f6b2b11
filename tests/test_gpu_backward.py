"""GPU parity of the backward pass (gqe_attn_prefill_backward, then
gqe_route_backward) against the oracle's backward on the same seeded inputs.

The small cases feed the oracle's routing (selection, gates and the position
lists built from it) to the GPU kernels, so both sides differentiate the same
routing: dQ, dK, dV and the router-logit gradient are compared element by
element.  The full-size dense_gqa case runs the GPU's own router first (every
head of a group is selected there, so the selections agree) and is checked on
what the oracle computes in seconds: the first 128 positions (dQ and the logit
gradients of a prefix do not depend on later positions), the last 8 key rows
of dK/dV and query rows of dQ (only query rows at or after them contribute),
and sum_s dK[b,s,q] = 0 everywhere (softmax shift invariance).

Tolerance: the forward's output tolerance, max-abs 2e-2 (bf16 inputs) or 1e-4
(fp32).  The gradients are accumulated in fp32 from the same inputs the oracle
reads, and the attention output is recomputed in fp32, so nothing on the GPU
side is rounded to bf16 after the inputs."""
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
    W["tiny_f32"],
    C("bw_k2_ragged", B=2, T=200, d_model=64, h=8, g=2, d_h=128, k=2, seed=91),
    C("bw_d64_k1", B=1, T=97, d_model=64, h=6, g=3, d_h=64, k=1, seed=92),
    C("bw_dense_k4", B=1, T=161, d_model=64, h=8, g=2, d_h=128, k=4, seed=93),
    C("bw_f32_d128", B=1, T=70, d_model=32, h=4, g=2, d_h=128, k=1, dtype="f32", seed=94),
    C("bw_T1", B=3, T=1, d_model=32, h=8, g=2, d_h=128, k=2, seed=95),
    C("bw_skew_h16", B=1, T=150, d_model=96, h=16, g=8, d_h=128, k=1, head0_bias=1.0, seed=96),
]


def _outputs(w, dev="cuda"):
    f32 = dict(dtype=torch.float32, device=dev)
    nan = float("nan")  # every element must be written
    return (torch.full((w.B, w.T, w.h, w.d_h), nan, **f32), torch.full((w.B, w.T, w.g, w.d_h), nan, **f32),
            torch.full((w.B, w.T, w.g, w.d_h), nan, **f32), torch.full((w.B, w.T, w.h), nan, **f32))


def gpu_backward_oracle_routing(w, inp, dO, idx_o, gate_o, idx_override=None):
    g = U.gqe()
    idx_d, offs, pos, chunk = U.oracle_tables(w, idx_o)
    if idx_override is not None:
        idx_d = idx_override.to("cuda")
    gate_d = torch.from_numpy(gate_o.astype(np.float32)).cuda()
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    dQ, dK, dV, dl = _outputs(w)
    ws = torch.zeros(g.gqe_backward_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    g.gqe_attn_prefill_backward(shape, U.to_dev(inp["Q"]), U.to_dev(inp["K"]), U.to_dev(inp["V"]), idx_d, gate_d,
                                offs, pos, chunk, U.to_dev(dO), dQ, dK, dV, dl, ws)
    torch.cuda.synchronize()
    st = g.gqe_get_device_status(ws)
    return [t.cpu().numpy().astype(np.float64) for t in (dQ, dK, dV, dl)], st


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_backward_small(w):
    inp = gqe_synth.make_inputs(w)
    dO = gqe_synth.make_output_grad(w)
    idx_o, gate_o, _, _ = U.oracle_route(w, inp)
    (dQ, dK, dV, dl), st = gpu_backward_oracle_routing(w, inp, dO, idx_o, gate_o)
    assert st == 0, f"device status {st}"
    want_q, want_k, want_v, dgate = oracle.attn_backward(inp["Q"], inp["K"], inp["V"], idx_o, gate_o,
                                                         dO.float().numpy())
    want_l, want_x, want_w, want_b = oracle.route_backward(inp["x"], inp["W_r"], idx_o, gate_o, dgate)
    tol = U.TOL[w.dtype]
    for name, got, want in (("dQ", dQ, want_q), ("dK", dK, want_k), ("dV", dV, want_v), ("dlogits", dl, want_l)):
        assert np.isfinite(got).all(), f"{w.name}: {name} has unwritten or non-finite elements"
        err = float(np.abs(got - want).max())
        assert err <= tol, f"{w.name}: {name} max abs error {err} (scale {np.abs(want).max():.3g})"
    # on through the router, from the GPU's own logit gradients
    dx, dW, db = gpu_route_backward(w, inp, torch.from_numpy(dl.astype(np.float32)))
    for name, got, want in (("dx", dx, want_x), ("dW_r", dW, want_w), ("dbias", db, want_b)):
        err = float(np.abs(got - want).max())
        assert err <= tol, f"{w.name}: {name} max abs error {err} (scale {np.abs(want).max():.3g})"


def gpu_route_backward(w, inp, dlogits):
    g = U.gqe()
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    nan = float("nan")
    f32 = dict(dtype=torch.float32, device="cuda")
    dx = torch.full((w.B, w.T, w.d_model), nan, **f32)
    dW = torch.full((w.d_model, w.h), nan, **f32)
    db = torch.full((w.h,), nan, **f32)
    ws = torch.zeros(g.gqe_backward_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    g.gqe_route_backward(shape, U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), dlogits.cuda(), dx, dW, db, ws)
    torch.cuda.synchronize()
    return [t.cpu().numpy().astype(np.float64) for t in (dx, dW, db)]


ROUTE_BWD_SMALL = [
    # two 32-head passes (dx summed over them), a ragged column block and token tile
    C("rb_h64_ragged", B=1, T=300, d_model=200, h=64, g=8, d_h=128, k=2, seed=97),
    C("rb_f32_h40", B=2, T=70, d_model=36, h=40, g=4, d_h=64, k=3, dtype="f32", seed=98),
]


@pytest.mark.parametrize("name", ["dense_gqa", "gqe_prefill"] + [w.name for w in ROUTE_BWD_SMALL])
def test_route_backward_full_size(name):
    """Router gradients from a seeded gate gradient: the oracle's logit
    gradients go in, dx, dW_r and dbias are compared in full (at full size,
    and on small shapes with more than 32 heads and ragged tiles)."""
    w = W[name] if name in W else next(x for x in ROUTE_BWD_SMALL if x.name == name)
    inp = gqe_synth.make_inputs(w)
    idx_o, gate_o, _, _ = U.oracle_route(w, inp)
    dgate = np.random.default_rng(w.seed + 7).standard_normal(idx_o.shape)
    want_l, want_x, want_w, want_b = oracle.route_backward(inp["x"], inp["W_r"], idx_o, gate_o, dgate)
    dx, dW, db = gpu_route_backward(w, inp, torch.from_numpy(want_l.astype(np.float32)))
    for nm, got, want in (("dx", dx, want_x), ("dW_r", dW, want_w), ("dbias", db, want_b)):
        assert np.isfinite(got).all(), f"{nm} has unwritten or non-finite elements"
        err = float(np.abs(got - want).max())
        assert err <= U.TOL["bf16"], f"{name}: {nm} max abs error {err} (scale {np.abs(want).max():.3g})"


def test_backward_reports_foreign_index():
    """An index outside its group is reported in the status word and skipped
    (no fault)."""
    w = SMALL[1]
    inp = gqe_synth.make_inputs(w)
    dO = gqe_synth.make_output_grad(w)
    idx_o, gate_o, _, _ = U.oracle_route(w, inp)
    bad = torch.from_numpy(idx_o.copy())
    bad[0, 5, 0, 0] = w.h - 1  # a head of the last group, in group 0's slot
    (dQ, dK, dV, dl), st = gpu_backward_oracle_routing(w, inp, dO, idx_o, gate_o, idx_override=bad)
    U.gqe()
    import routed_head_gqa_b200 as g

    assert st == g.GQE_ERR_INVALID_ARGUMENT


def test_backward_dense_gqa_full_size():
    w = W["dense_gqa"]
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    dO = gqe_synth.make_output_grad(w)
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, "cuda")
    buf.route(U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]))
    dQ, dK, dV, dl = buf.backward(U.to_dev(inp["Q"]), U.to_dev(inp["K"]), U.to_dev(inp["V"]), U.to_dev(dO))
    torch.cuda.synchronize()
    assert buf.backward_status() == 0
    dQ, dK, dV, dl = (t.cpu().numpy().astype(np.float64) for t in (dQ, dK, dV, dl))
    for name, a in (("dQ", dQ), ("dK", dK), ("dV", dV), ("dlogits", dl)):
        assert np.isfinite(a).all(), f"{name} has non-finite elements"
    tol = U.TOL["bf16"]
    idx_o, gate_o, _, _ = U.oracle_route(w, inp)
    dOn = dO.float().numpy()
    # prefix: the first Tp positions
    Tp = 128
    pq, _, _, pg = oracle.attn_backward(inp["Q"][:, :Tp].contiguous(), inp["K"][:, :Tp].contiguous(),
                                        inp["V"][:, :Tp].contiguous(), idx_o[:, :Tp], gate_o[:, :Tp],
                                        dOn[:, :Tp])
    pl = oracle.route_backward(inp["x"][:, :Tp].contiguous(), inp["W_r"], idx_o[:, :Tp], gate_o[:, :Tp], pg)[0]
    for name, got, want in (("dQ prefix", dQ[:, :Tp], pq), ("dlogits prefix", dl[:, :Tp], pl)):
        err = float(np.abs(got - want).max())
        assert err <= tol, f"{name}: max abs error {err}"
    # suffix: key rows and query rows at or after T - 8
    t0 = w.T - 8
    sq, sk, sv, _ = oracle.attn_backward(inp["Q"], inp["K"], inp["V"], idx_o, gate_o, dOn, t_min=t0)
    for name, got, want in (("dQ suffix", dQ[:, t0:], sq[:, t0:]), ("dK suffix", dK[:, t0:], sk[:, t0:]),
                            ("dV suffix", dV[:, t0:], sv[:, t0:])):
        err = float(np.abs(got - want).max())
        assert err <= tol, f"{name}: max abs error {err}"
    # softmax shift invariance: the score gradients of every row sum to zero.  dK
    # accumulates dS rounded to bf16 on the tensor cores, so each row's sum over
    # its keys carries about 2^-9 |dS| sqrt(n) of rounding, and the invariant
    # holds to the element tolerance, not tighter.
    assert np.abs(dK.sum(axis=1)).max() <= tol, "sum_s dK != 0"
    # and every group's logit gradients sum to zero
    assert np.abs(dl.reshape(w.B, w.T, w.g, -1).sum(-1)).max() <= 1e-4


@pytest.mark.parametrize("w", [SMALL[1], SMALL[3], W["dense_gqa"]], ids=lambda w: w.name)
def test_train_forward_and_saved_backward(w):
    """gqe_attn_prefill_train: O within the forward tolerance of the oracle and
    O32 * gate equal to it within the same bound (the ungated rows it saves);
    gqe_attn_prefill_backward_saved on those statistics gives gradients
    bit-identical to gqe_attn_prefill_backward, which recomputes them."""
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    dO = gqe_synth.make_output_grad(w).cuda()
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, "cuda")
    buf.route(U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]))
    Q, K, V = (U.to_dev(inp[n]) for n in ("Q", "K", "V"))
    O32 = torch.full((w.B, w.T, w.h, w.d_h), float("nan"), device="cuda")
    lse = torch.full((w.B, w.T, w.h), float("nan"), device="cuda")
    g.gqe_attn_prefill_train(shape, Q, K, V, buf.idx, buf.gate, buf.head_offsets, buf.head_pos,
                             buf.head_chunk_offsets, buf.O, O32, lse, buf.workspace)
    torch.cuda.synchronize()
    assert buf.status() == 0
    excl, idx_o, gate_o = U.check_routing(w, inp, buf.idx, buf.gate)
    rows = U.cover_rows(w, idx_o, U.sm_count(), n_min=512) if w.T > 512 else None
    err, n = U.compare_rows(w, inp, buf.O, idx_o, gate_o, excl, rows)
    assert err <= U.TOL["bf16"], f"{w.name}: training forward O error {err}"
    sel = torch.zeros((w.B, w.T, w.h), dtype=torch.bool, device="cuda")
    sel.scatter_(2, buf.idx.reshape(w.B, w.T, -1).long(), True)
    gates = torch.zeros((w.B, w.T, w.h), device="cuda").scatter_(2, buf.idx.reshape(w.B, w.T, -1).long(),
                                                                  buf.gate.reshape(w.B, w.T, -1))
    gated = (O32 * gates[..., None])[sel]
    assert torch.isfinite(O32[sel]).all() and torch.isfinite(lse[sel]).all()
    assert (gated - buf.O.float()[sel]).abs().max().item() <= U.TOL["bf16"]
    outs = []
    for saved in (False, True):
        f32 = dict(dtype=torch.float32, device="cuda")
        dQ, dK, dV = (torch.full(sh, float("nan"), **f32) for sh in
                      ((w.B, w.T, w.h, w.d_h), (w.B, w.T, w.g, w.d_h), (w.B, w.T, w.g, w.d_h)))
        dl = torch.full((w.B, w.T, w.h), float("nan"), **f32)
        ws = torch.zeros(g.gqe_backward_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
        args = (shape, Q, K, V, buf.idx, buf.gate, buf.head_offsets, buf.head_pos, buf.head_chunk_offsets, dO)
        if saved:
            g.gqe_attn_prefill_backward_saved(*args, O32, lse, dQ, dK, dV, dl, ws)
        else:
            g.gqe_attn_prefill_backward(*args, dQ, dK, dV, dl, ws)
        torch.cuda.synchronize()
        assert g.gqe_get_device_status(ws) == 0
        outs.append((dQ, dK, dV, dl))
    for name, a, b in zip(("dQ", "dK", "dV", "dlogits"), outs[0], outs[1]):
        assert torch.equal(a, b), f"{w.name}: {name} differs between the saved and the recomputing backward"
