"""GPU unit checks of the tensor-core building blocks (TMA + 128B swizzle,
UMMA smem descriptors K-major / MN-major, A operand from TMEM, TMEM loads) and
of the bounded-wait failure path, against plain torch matmuls."""
import ctypes
import os

import pytest
import torch

from routed_head_gqa_b200 import build as gqe_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def selftest():
    gqe_build.build()
    lib = ctypes.CDLL(gqe_build.SELFTEST_LIB)
    lib.gqe_selftest_umma_tile.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 5
    lib.gqe_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.gqe_selftest_exp2_poly.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    return lib


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["ss_kmajor", "ss_mnmajor_b", "ts_tmem_a"])
def test_umma_tile(selftest, mode):
    g = torch.Generator(device="cuda").manual_seed(mode)
    A = torch.randn(128, 128, device="cuda", generator=g).to(torch.bfloat16)
    Bm = torch.randn(128, 128, device="cuda", generator=g).to(torch.bfloat16)
    C = torch.full((128, 128), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert selftest.gqe_selftest_umma_tile(mode, A.data_ptr(), Bm.data_ptr(), C.data_ptr(), status.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = A.float() @ (Bm.float().t() if mode == 0 else Bm.float())
    err = (C - ref).abs().max().item()
    assert err < 1e-2, f"mode {mode}: max error {err}"


def test_bounded_wait_times_out(selftest):
    """A wait on a barrier that nothing completes returns an error status
    (after about 2 s) instead of hanging the GPU; the context stays usable."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert selftest.gqe_selftest_wait_timeout(status.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 4  # GQE_ERR_DEVICE_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0


def test_exp2_poly_bound(selftest):
    """The softmax's FMA-pipe 2^x against the exact power of two (float64):
    relative error within the fit's 1.2e-4 bound over [-126, 8] (a dense sweep
    plus every integer and half-integer, where the range reduction switches),
    exact at the integers (p(0) = 1), and the clamp: inputs at or below -126
    (down to -inf) give 2^-126, a value that vanishes next to a row sum >= 1."""
    import numpy as np

    sweep = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64)
    ints = np.arange(-126, 9, dtype=np.float64)
    halves = np.concatenate([ints[:-1] + 0.5, ints[:-1] + 0.5 - 2.0 ** -20, ints[:-1] + 0.5 + 2.0 ** -20])
    x = np.concatenate([sweep, ints, halves]).astype(np.float32)
    low = np.array([-126.25, -126.5, -127.0, -149.0, -1e4, -np.inf], dtype=np.float32)
    xs = torch.from_numpy(np.concatenate([x, low])).cuda()
    ys = torch.empty_like(xs)
    s = torch.cuda.current_stream().cuda_stream
    assert selftest.gqe_selftest_exp2_poly(xs.data_ptr(), ys.data_ptr(), xs.numel(), s) == 0
    torch.cuda.synchronize()
    y = ys.cpu().numpy().astype(np.float64)
    n = x.size
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y[:n] / exact - 1.0)
    assert rel.max() <= 1.2e-4, f"max relative error {rel.max():.3e} at x={x[rel.argmax()]}"
    at_ints = y[sweep.size:sweep.size + ints.size]
    assert np.array_equal(at_ints, np.exp2(ints)), "2^n not exact at integer n"
    tail = y[n:]
    assert np.all(tail == 2.0 ** -126), tail
