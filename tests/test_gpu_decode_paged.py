"""GPU parity of the paged decode (gqe_attn_decode_paged) against the CPU
oracle's paged decode on the same seeded pages (max-abs 2e-2 bf16 / 1e-4
fp32), and bit-equality with the contiguous GPU decode of the same cache."""
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
    (C("pg_bf16_ps16", B=5, T=1, d_model=64, h=8, g=2, d_h=128, k=2, decode=True, Lmin=1, Lmax=704, seed=51), 16),
    (C("pg_bf16_ps1", B=3, T=1, d_model=64, h=8, g=4, d_h=64, k=1, decode=True, Lmin=1, Lmax=96, seed=52), 1),
    (C("pg_f32_ps64", B=4, T=1, d_model=32, h=4, g=2, d_h=32, k=2, dtype="f32", decode=True, Lmin=1, Lmax=320,
       seed=53), 64),
    (W["gqe_decode"], 256),
]


@pytest.mark.parametrize("w,ps", CASES, ids=[f"{c[0].name}-ps{c[1]}" for c in CASES])
def test_decode_paged(w, ps):
    g = U.gqe()
    inp = gqe_synth.make_inputs(w)
    Kp, Vp, bt = gqe_synth.make_paged_cache(inp["K_cache"], inp["V_cache"], ps)
    shape = g.make_shape(w.B, 1, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, "cuda", Lmax=w.Lmax)
    buf.route(U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]))
    lengths = U.to_dev(inp["lengths"])
    Op = torch.empty_like(buf.O)
    g.gqe_attn_decode_paged(shape, U.to_dev(inp["q"]), U.to_dev(Kp), U.to_dev(Vp), ps, U.to_dev(bt), lengths,
                            buf.idx, buf.gate, Op, buf.workspace)
    buf.decode(U.to_dev(inp["q"]), U.to_dev(inp["K_cache"]), U.to_dev(inp["V_cache"]), lengths)
    torch.cuda.synchronize()
    assert buf.status() == 0
    # the same kernel arithmetic whether the rows are paged or contiguous
    assert torch.equal(Op, buf.O), "paged decode differs from the contiguous decode"
    excl, idx_o, gate_o = U.check_routing(w, inp, buf.idx, buf.gate)
    want = oracle.decode_paged(inp["q"], Kp, Vp, bt, inp["lengths"], idx_o, gate_o)
    got = Op.float().reshape(w.B, w.h, w.d_h).cpu().numpy()
    keep = ~excl.reshape(-1)
    err = float(np.abs(got[keep] - want[keep]).max())
    assert err <= U.TOL[w.dtype], f"{w.name}: paged decode max abs error {err}"
