"""The work counts behind the roofline figures (routed_head_gqa_b200.metrics),
pinned to the pages and to a realised routing (CPU)."""
import os

import numpy as np
import torch

import oracle
from routed_head_gqa_b200 import metrics

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            rows.append([int(v) for v in line.split()])
    return rows


def dense_flops(B, T, h, d_h):
    """Causal attention of all h query heads: 4*d_h FLOPs per visible (query, key) pair."""
    return 4 * d_h * B * h * (T * (T + 1) // 2)


def test_active_fraction_golden():
    """Routed heads plus the shared head run 9 of 16 query-head computations,
    about 56 % of the dense query-side work."""
    h, g, k, shared, active, pct = read_golden("active_fraction.txt")[0]
    B, T, d_h = 2, 4096, 128
    routed = metrics.prefill_active_flops(B, T, g, k, d_h)
    shared_flops = shared * metrics.prefill_active_flops(B, T, 1, 1, d_h)  # one head per token
    frac = (routed + shared_flops) / dense_flops(B, T, h, d_h)
    assert routed + shared_flops == active * dense_flops(B, T, 1, d_h)
    assert round(100 * frac) == pct, f"{100 * frac:.2f} % of the dense work, the page says about {pct} %"


def test_active_flops_match_a_realised_routing():
    """The closed form equals the count taken from the oracle's routing of a
    random input (every token selects exactly k heads per group)."""
    rng = np.random.default_rng(7)
    B, T, d_model, h, g, k, d_h = 2, 37, 24, 16, 4, 3, 64
    x = rng.standard_normal((B * T, d_model)).astype(np.float32)
    W = rng.standard_normal((d_model, h)).astype(np.float32)
    idx, _, _, _ = oracle.route(x, W, h, g, k)
    idx = torch.from_numpy(np.asarray(idx).reshape(B, T, g, k))
    assert metrics.prefill_active_flops_from_routing(idx, d_h) == metrics.prefill_active_flops(B, T, g, k, d_h)

