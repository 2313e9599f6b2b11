"""Host-side helpers the GPU tests rely on, checked on the CPU: the routing
tables built from the oracle's selection (position lists and per-32-position
chunk starts) against a direct enumeration, and the seeded generators'
determinism and shapes."""
import numpy as np
import torch

import gqe_synth
import oracle
from tests import gpu_util as U


def test_oracle_tables_match_enumeration():
    w = gqe_synth.custom("tables", B=2, T=77, d_model=16, h=6, g=3, d_h=32, k=1, seed=7)
    inp = gqe_synth.make_inputs(w)
    idx_o, _, _, _ = oracle.route(inp["x"], inp["W_r"], w.h, w.g, w.k)
    idx_d, offs, pos, chunk = (t.numpy() for t in U.oracle_tables(w, idx_o, dev="cpu"))
    assert np.array_equal(idx_d, idx_o)
    nchunk = (w.T + 31) // 32
    for b in range(w.B):
        for j in range(w.h):
            bj = b * w.h + j
            want = [t for t in range(w.T) if j in idx_o[b, t].reshape(-1)]
            assert list(pos[offs[bj]:offs[bj + 1]]) == want
            for c in range(nchunk):
                first = next((e for e in range(offs[bj], offs[bj + 1]) if pos[e] >= 32 * c), offs[bj + 1])
                assert chunk[bj * nchunk + c] == first
    assert offs[-1] == w.B * w.T * w.g * w.k


def test_output_grad_is_seeded():
    w = gqe_synth.custom("grad", B=1, T=5, d_model=8, h=4, g=2, d_h=32, k=1, seed=3)
    a, b = gqe_synth.make_output_grad(w), gqe_synth.make_output_grad(w)
    assert a.shape == (1, 5, 4, 32) and a.dtype == torch.bfloat16
    assert torch.equal(a, b)
    other = gqe_synth.make_output_grad(gqe_synth.custom("grad", B=1, T=5, d_model=8, h=4, g=2, d_h=32, k=1, seed=4))
    assert not torch.equal(a, other)
