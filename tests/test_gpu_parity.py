"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Tolerances: routing exact (tokens with an oracle top-k
margin below 1e-5 excluded and counted), gates 1e-5, outputs max-abs 1e-4
(fp32) / 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import gqe_synth
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

W = gqe_synth.WORKLOADS
C = gqe_synth.custom

# Small prefill cases: several 128-row tiles and KV tiles, ragged tails, the
# degenerate group shapes (MHA g=h, MQA g=1), k = h/g (dense GQA up to the
# gates), T = 1, a skewed router.
SMALL_BF16 = [
    C("bf16_k1", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=1, seed=11),
    C("bf16_k2", B=2, T=300, d_model=64, h=8, g=2, d_h=128, k=2, seed=12),
    C("bf16_k3", B=1, T=170, d_model=64, h=8, g=2, d_h=128, k=3, seed=13),
    C("bf16_dense_k4", B=1, T=257, d_model=64, h=8, g=2, d_h=128, k=4, seed=14),
    C("bf16_mha", B=1, T=200, d_model=64, h=4, g=4, d_h=128, k=1, seed=15),
    C("bf16_mqa_all", B=1, T=160, d_model=64, h=4, g=1, d_h=128, k=4, seed=16),
    C("bf16_mqa_k2", B=1, T=190, d_model=64, h=4, g=1, d_h=128, k=2, seed=17),
    C("bf16_T1", B=3, T=1, d_model=64, h=8, g=2, d_h=128, k=2, seed=18),
    C("bf16_T33", B=2, T=33, d_model=64, h=8, g=2, d_h=128, k=2, seed=19),
    C("bf16_T129", B=1, T=129, d_model=64, h=8, g=2, d_h=128, k=1, seed=20),
    C("bf16_skew", B=1, T=520, d_model=96, h=16, g=8, d_h=128, k=1, head0_bias=1.0, seed=21),
    # Router and compaction shapes: d_model split over 4-CTA clusters (8 k-blocks,
    # 2 token tiles); 64, 128 and 256 heads (one, two and four 64-head MMA blocks;
    # a head scan over several 32-head rounds); T not a multiple of 32 (counts from
    # the separate pass).
    C("bf16_route_ks4", B=1, T=256, d_model=512, h=32, g=8, d_h=128, k=2, seed=22),
    C("bf16_h64", B=2, T=96, d_model=256, h=64, g=8, d_h=128, k=2, seed=23),
    C("bf16_h128", B=1, T=64, d_model=128, h=128, g=16, d_h=128, k=1, seed=24),
    C("bf16_h256_T40", B=1, T=40, d_model=128, h=256, g=32, d_h=128, k=3, seed=25),
    # Split-KV: so few units that each is split over its KV tiles and merged by
    # log-sum-exp (32 units of up to 16 KV tiles -> 8 splits; 5 units over a
    # ragged T -> 4 splits)
    C("bf16_splitkv_k2", B=1, T=2048, d_model=64, h=8, g=2, d_h=128, k=2, seed=26),
    C("bf16_splitkv_ragged", B=1, T=1100, d_model=64, h=4, g=1, d_h=128, k=1, seed=27),
]
SMALL_F32 = [
    W["tiny_f32"],
    C("f32_d64_k2", B=2, T=100, d_model=48, h=8, g=2, d_h=64, k=2, dtype="f32", seed=31),
    C("f32_d128_mha", B=1, T=70, d_model=32, h=4, g=4, d_h=128, k=1, dtype="f32", seed=32),
    C("f32_T1", B=2, T=1, d_model=32, h=4, g=2, d_h=32, k=1, dtype="f32", seed=33),
]


@pytest.mark.parametrize("w", SMALL_BF16 + SMALL_F32, ids=lambda w: w.name)
def test_prefill_small(w):
    err, n, excl = U.prefill_parity(w)
    assert n > 0
    assert err <= U.TOL[w.dtype], f"{w.name}: max abs error {err} over {n} rows ({excl} tokens excluded)"


@pytest.mark.parametrize("name", ["dense_gqa", "gqe_prefill", "gqe_long"])
def test_prefill_full_size_covered(name):
    """Full-size workloads in the benchmark's launch configuration.  The oracle
    computes at least 4096 rows, chosen to reach every path of the persistent
    kernel: whole work units (every position of each, all heads) that a first,
    a middle and the last CTA run first, midway and last, every sequence's last
    window, the most skewed windows, and random rows."""
    w = W[name]
    err, n, excl = U.prefill_parity(w, cover=True)
    assert n >= 4096 - 64, f"{name}: only {n} rows compared"
    assert err <= U.TOL[w.dtype], f"{name}: max abs error {err} over {n} rows ({excl} tokens excluded)"


def test_prefill_32k_sampled():
    """A 32768-token sequence (B=1, h=16, g=8, k=1): every position of the last
    window and of the windows that the first and the last CTA run first, and
    random rows, 1024 rows in all (the oracle's cost grows with the context)."""
    w = W["gqe_32k"]
    inp = gqe_synth.make_inputs(w)
    buf = U.run_prefill(w, inp)
    excl, idx_o, gate_o = U.check_routing(w, inp, buf.idx, buf.gate)
    _, nwin = U.prefill_windows(w)
    span = 2 * 32 * (4 // w.k)
    rows = set(range(w.T - span, w.T))
    for c in (0, min(w.B * w.g * nwin, U.sm_count()) - 1):
        b, _, win = U.cta_units(w, U.sm_count(), c)[0]
        rows.update(range(b * w.T + win * span, b * w.T + min((win + 1) * span, w.T)))
    rng = np.random.default_rng(32768)
    rows.update(int(r) for r in rng.choice(w.B * w.T, 1024 - len(rows), replace=False))
    err, n = U.compare_rows(w, inp, buf.O, idx_o, gate_o, excl, np.array(sorted(rows)))
    assert n >= 900 and err <= U.TOL["bf16"], f"gqe_32k: max abs error {err} over {n} rows"


def test_full_size_repeatable():
    """Routing and prefill at the gqe_prefill size (the bench's launch
    configuration) run twice on the same inputs give bit-identical tables and
    outputs."""
    w = W["gqe_prefill"]
    inp = gqe_synth.make_inputs(w)
    a = U.run_prefill(w, inp)
    first = [t.clone() for t in (a.idx, a.gate, a.head_offsets, a.head_pos, a.head_chunk_offsets, a.O)]
    a.O.fill_(float("nan"))
    a.route(U.to_dev(inp["x"]), U.to_dev(inp["W_r"]), U.to_dev(inp["bias"]))
    a.prefill(U.to_dev(inp["Q"]), U.to_dev(inp["K"]), U.to_dev(inp["V"]))
    torch.cuda.synchronize()
    assert a.status() == 0
    second = (a.idx, a.gate, a.head_offsets, a.head_pos, a.head_chunk_offsets, a.O)
    for name, x, y in zip(("idx", "gate", "head_offsets", "head_pos", "head_chunk_offsets", "O"), first, second):
        assert torch.equal(x, y), f"{name} differs between two runs"


SMALL_DECODE = [
    C("dec_bf16_small", B=5, T=1, d_model=64, h=8, g=2, d_h=128, k=2, decode=True, Lmin=1, Lmax=700, seed=41),
    C("dec_bf16_d64", B=3, T=1, d_model=64, h=8, g=4, d_h=64, k=1, decode=True, Lmin=200, Lmax=513, seed=42),
    C("dec_f32_d32", B=4, T=1, d_model=32, h=4, g=2, d_h=32, k=2, dtype="f32", decode=True, Lmin=1, Lmax=300,
      seed=43),
    C("dec_bf16_k4", B=2, T=1, d_model=64, h=8, g=2, d_h=128, k=4, decode=True, Lmin=1000, Lmax=1300, seed=44),
]


@pytest.mark.parametrize("w", SMALL_DECODE + [W["gqe_decode"]], ids=lambda w: w.name)
def test_decode(w):
    err, n, excl = U.decode_parity(w)
    assert err <= U.TOL[w.dtype], f"{w.name}: max abs error {err} ({excl} sequences excluded)"


def test_decode_length_edges():
    """lengths of exactly 1 and exactly Lmax."""
    w = C("dec_edges", B=2, T=1, d_model=64, h=8, g=2, d_h=128, k=2, decode=True, Lmin=1, Lmax=300, seed=45)
    inp = gqe_synth.make_inputs(w)
    inp["lengths"] = torch.tensor([1, 300], dtype=torch.int32)
    for name in ("K_cache", "V_cache"):
        inp[name][1] = torch.randn(300, w.g, w.d_h, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    buf = U.run_decode(w, inp)
    excl, idx_o, gate_o = U.check_routing(w, inp, buf.idx, buf.gate)
    import oracle

    want = oracle.decode(inp["q"], inp["K_cache"], inp["V_cache"], inp["lengths"], idx_o, gate_o)
    got = buf.O.float().reshape(w.B, w.h, w.d_h).cpu().numpy()
    assert np.abs(got - want)[~excl.reshape(-1)].max() <= U.TOL["bf16"]


def test_prefill_repeatable():
    """Two runs on the same inputs give bit-identical outputs (no races)."""
    w = SMALL_BF16[1]
    inp = gqe_synth.make_inputs(w)
    a = U.run_prefill(w, inp)
    O1 = a.O.clone()
    a.prefill(U.to_dev(inp["Q"]), U.to_dev(inp["K"]), U.to_dev(inp["V"]))
    torch.cuda.synchronize()
    assert torch.equal(O1, a.O)
