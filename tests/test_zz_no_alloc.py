"""gqe_route_static: the routing entry point for callers that cannot allocate
device memory (an arena-planned serving runtime, code that may not call
cudaMalloc or an allocating library where it runs).  It keeps its scratch in
an array owned by the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different shapes,
and checks each result against gqe_route on the same inputs (routing is
compared exactly, gates within the 1e-5 used by the other tests).  This file
is collected last, so a run that stops at its first failure has already run
every other test; the test also passes on its own in a fresh process."""
import ctypes

import pytest
import torch

import gqe_synth
from routed_head_gqa_b200 import build as gqe_build

CASES = [
    gqe_synth.custom("static_a", B=8, T=4096, d_model=512, h=32, g=8, d_h=128, k=2, seed=61),
    gqe_synth.custom("static_b", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=1, head0_bias=0.5, seed=62),
]


def _outputs(w, dev):
    g_, k = w.g, w.k
    import routed_head_gqa_b200 as g

    return {
        "idx": torch.empty((w.B, w.T, g_, k), dtype=torch.int32, device=dev),
        "gate": torch.empty((w.B, w.T, g_, k), dtype=torch.float32, device=dev),
        "head_offsets": torch.empty(w.B * w.h + 1, dtype=torch.int32, device=dev),
        "head_pos": torch.empty(w.B * w.T * g_ * k, dtype=torch.int32, device=dev),
        "head_chunk_offsets": torch.empty(w.B * w.h * g.gqe_chunk_count(w.T), dtype=torch.int32, device=dev),
    }


@pytest.mark.gpu
def test_route_static_matches_route_twice():
    gqe_build.build()
    import routed_head_gqa_b200 as g

    dev = torch.device("cuda", 0)
    for w in CASES:  # two calls in a row; the second finds the first one's counts in the shared scratch
        inp = gqe_synth.make_inputs(w)
        x, W_r = inp["x"].to(dev), inp["W_r"].to(dev)
        bias = inp["bias"].to(dev) if inp["bias"] is not None else None
        shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, torch.bfloat16)
        ref = g.Buffers(shape, dev)
        ref.route(x, W_r, bias)
        out = _outputs(w, dev)
        rc = g._lib.gqe_route_static(ctypes.byref(shape), x.data_ptr(), W_r.data_ptr(),
                                     bias.data_ptr() if bias is not None else None, out["idx"].data_ptr(),
                                     out["gate"].data_ptr(), out["head_offsets"].data_ptr(),
                                     out["head_pos"].data_ptr(), out["head_chunk_offsets"].data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
        assert rc == g.GQE_OK, g.gqe_status_string(rc)
        torch.cuda.synchronize()
        st = g.gqe_route_static_status()  # the array's own status word: no expired wait, no bad counts
        assert st == g.GQE_OK, g.gqe_status_string(st)
        assert torch.equal(out["idx"], ref.idx), w.name
        assert (out["gate"] - ref.gate).abs().max().item() <= 1e-5, w.name
        assert torch.equal(out["head_offsets"], ref.head_offsets), w.name
        assert torch.equal(out["head_pos"], ref.head_pos), w.name
        assert torch.equal(out["head_chunk_offsets"], ref.head_chunk_offsets), w.name


def test_route_static_rejects_shapes_beyond_its_scratch():
    """B * h * ceil(T/32) above 1,048,576 counts: GQE_ERR_SCRATCH_LIMIT, nothing enqueued."""
    import routed_head_gqa_b200 as g

    gqe_build.build()
    s = g.make_shape(64, 32768, 128, 64, 8, 128, 2, g.GQE_BF16)  # 64*64*1024 counts
    fake = 0x10000  # never dereferenced: the size check fails first
    rc = g._lib.gqe_route_static(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, fake, None)
    assert rc == g.GQE_ERR_SCRATCH_LIMIT
    assert g.gqe_status_string(rc) == "GQE_ERR_SCRATCH_LIMIT"
