"""Property sweep of the oracle's router and compaction over random shapes
(CPU): per (token, group) the selection equals the brute-force best k-subset
with ties to the lower index, the gates are the softmax of the selected logits,
the margin is l_(k) - l_(k+1), and the compaction lists are np.nonzero of the
selection mask.  Shapes include one head per group (h = g), k = h/g, ragged T
(not a multiple of the 32-token chunk) and heavily tied logits."""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
from scipy.special import softmax

import oracle
from tests.oracle_pins import _bruteforce_select


@st.composite
def shapes(draw):
    g = draw(st.integers(1, 4))
    hpg = draw(st.integers(1, 6))
    k = draw(st.integers(1, hpg))
    B = draw(st.integers(1, 3))
    T = draw(st.integers(1, 70))
    d_model = draw(st.integers(1, 24))
    ties = draw(st.booleans())
    seed = draw(st.integers(0, 2**31 - 1))
    return B, T, g * hpg, g, k, d_model, ties, seed


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(shapes())
def test_route_and_compact_properties(shape):
    B, T, h, g, k, d_model, ties, seed = shape
    hpg = h // g
    rng = np.random.default_rng(seed)
    if ties:
        # small integers: many exactly equal logits
        x = rng.integers(-1, 2, size=(B * T, d_model)).astype(np.float32)
        W = rng.integers(-1, 2, size=(d_model, h)).astype(np.float32)
    else:
        x = rng.standard_normal((B * T, d_model)).astype(np.float32)
        W = rng.standard_normal((d_model, h)).astype(np.float32)
    idx, gate, logits, margin = oracle.route(x, W, h, g, k)
    idx = np.asarray(idx).reshape(B * T, g, k)
    gate = np.asarray(gate).reshape(B * T, g, k)
    for r in range(B * T):
        for q in range(g):
            lg = logits[r, q * hpg:(q + 1) * hpg]
            want = [q * hpg + i for i in _bruteforce_select(lg, k)]
            assert list(idx[r, q]) == want
            sel = logits[r, idx[r, q]].astype(np.float64)
            assert np.allclose(gate[r, q], softmax(sel), rtol=0, atol=1e-14)
            srt = np.sort(lg.astype(np.float64))[::-1]
            assert margin[r, q] == (math.inf if k == hpg else srt[k - 1] - srt[k])
    offs, pos = oracle.compact(idx.reshape(B, T, g, k), h, g, k)
    mask = np.zeros((B, T, h), bool)
    for b in range(B):
        for t in range(T):
            mask[b, t, idx[b * T + t].reshape(-1)] = True
    assert offs[0] == 0 and offs[-1] == B * T * g * k
    for b in range(B):
        for j in range(h):
            assert np.array_equal(pos[offs[b * h + j]:offs[b * h + j + 1]], np.nonzero(mask[b, :, j])[0])
