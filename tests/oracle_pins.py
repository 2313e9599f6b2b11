"""Pins for the CPU oracle: facts fixed by the pages and by mathematics,
independent of the oracle's own code.

Every check takes an ``oracle.Oracle`` instance and raises AssertionError on a
mismatch, so the same checks run against the real oracle (test_oracle_pins.py)
and against deliberately broken copies of it (test_oracle_mutants.py).

Sources of the pinned facts:
  * torch.nn.functional.scaled_dot_product_attention (fp64, CPU, causal,
    enable_gqa) -- a library routine that expands KV heads by repetition
    like the ml-canon "56 GQA / MQA" page, section "PyTorch GQA", and scales
    by 1/sqrt(d) like IBM's GQA page (scaled dot-product attention).
  * freenetmedia.pl "Grouped-Query Attention", section "Jak dzialaja...":
    8 query heads in 2 groups -> heads 0-3 share KV head 0, heads 4-7 KV head 1
    (tests/golden/head_group_map.txt).
  * gist.science "Grouped Query Experts", "Resultats Experimentaux": with 16
    query heads, 8 KV groups and k=1, 8 routed query-head computations per
    token (tests/golden/active_heads.txt).
  * Brute force over all C(h/g, k) subsets for the top-k selection; closed
    forms (T=1, zero keys, constant values, one dominant key, k=2 gate =
    logistic of the logit gap, W_r=0 ties).
"""
from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import expit, softmax

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(shape, seed, scale=1.0):
    return (_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def read_golden(name):
    """Rows of integers from a golden fixture (lines starting with # are comments)."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(v) for v in line.split()])
    return rows


# --------------------------------------------------------------------------
# Router
# --------------------------------------------------------------------------

def check_router_onehot(o):
    """x = e_i gives logits = fp32(W_r[i, :] + bias): pins the orientation of
    W_r ([d_model, h]) and the bias term."""
    d_model, h, g = 6, 4, 2
    W = _f32((d_model, h), 1)
    bias = _f32((h,), 2)
    x = np.eye(d_model, dtype=np.float32)
    _, _, logits, _ = o.route(x, W, h, g, 1, bias=bias)
    expect = (W.astype(np.float64) + bias.astype(np.float64)).astype(np.float32)
    assert np.array_equal(logits, expect), "one-hot logits differ from W_r rows + bias"
    # doubling x doubles every logit exactly (linear, no constant term besides bias)
    x2 = _f32((5, d_model), 3)
    _, _, l1, _ = o.route(x2, W, h, g, 1)
    _, _, l2, _ = o.route(2 * x2, W, h, g, 1)
    assert np.array_equal(2 * l1, l2), "router is not linear in x"


def _bruteforce_select(lg, k):
    """Subset of size k with the largest exact logit sum; equal sums -> the
    lexicographically smallest index tuple.  Returned in (logit desc, index asc) order."""
    best, best_sum = None, None
    for comb in itertools.combinations(range(len(lg)), k):
        s = sum(Fraction(float(lg[i])) for i in comb)
        if best is None or s > best_sum:
            best, best_sum = comb, s
    return sorted(best, key=lambda i: (-float(lg[i]), i))


def check_router_bruteforce(o):
    """Selected heads equal the brute-force best subset per (token, group),
    including heavy ties (logits drawn from 3 values)."""
    for (h, g, k, seed, quant) in [(8, 2, 1, 10, False), (8, 2, 2, 11, False), (12, 3, 3, 12, False),
                                   (8, 2, 2, 13, True), (12, 2, 4, 14, True), (6, 6, 1, 15, False)]:
        hpg = h // g
        d_model = 16
        if quant:
            # one-hot tokens and a W_r with values in {-1, 0, 1}: many exact ties
            W = _rng(seed).integers(-1, 2, size=(d_model, h)).astype(np.float32)
            x = np.eye(d_model, dtype=np.float32)
        else:
            W = _f32((d_model, h), seed, 0.5)
            x = _f32((20, d_model), seed + 100)
        idx, gate, logits, margin = o.route(x, W, h, g, k)
        for r in range(x.shape[0]):
            for q in range(g):
                lg = logits[r, q * hpg:(q + 1) * hpg]
                want = [q * hpg + i for i in _bruteforce_select(lg, k)]
                assert list(idx[r, q]) == want, f"selection {list(idx[r, q])} != brute force {want}"
                srt = np.sort(lg.astype(np.float64))[::-1]
                exp_margin = math.inf if k == hpg else srt[k - 1] - srt[k]
                assert margin[r, q] == exp_margin, "margin is not l_(k) - l_(k+1)"


def check_router_zero_weights(o):
    """W_r = 0: every logit ties, so the first k heads of every group win and
    each gate is exactly 1/k."""
    h, g, k = 12, 3, 2
    x = _f32((7, 10), 5)
    idx, gate, _, _ = o.route(x, np.zeros((10, h), np.float32), h, g, k)
    hpg = h // g
    for q in range(g):
        assert (idx[:, q, :] == np.arange(q * hpg, q * hpg + k)).all(), "tie rule: lower index first"
    assert (gate == 1.0 / k).all(), "tied gates must be exactly 1/k"


def check_gates(o):
    """Gates are the router softmax renormalised over the k selected heads."""
    x = _f32((30, 16), 21)
    W = _f32((16, 8), 22, 0.7)
    # k = 1: gate is exactly 1
    _, gate1, _, _ = o.route(x, W, 8, 2, 1)
    assert (gate1 == 1.0).all(), "k=1 gates must be 1"
    # k = 2: gate of the top head is the logistic function of the logit gap
    idx, gate, logits, _ = o.route(x, W, 8, 2, 2)
    for r in range(x.shape[0]):
        for q in range(2):
            l0 = float(logits[r, idx[r, q, 0]])
            l1 = float(logits[r, idx[r, q, 1]])
            assert abs(gate[r, q, 0] - expit(l0 - l1)) < 1e-14
            assert abs(gate[r, q, 1] - expit(l1 - l0)) < 1e-14
    # k = 3 of 4: scipy softmax over the selected logits
    idx, gate, logits, _ = o.route(x, W, 8, 2, 3)
    for r in range(x.shape[0]):
        for q in range(2):
            sel = logits[r, idx[r, q]].astype(np.float64)
            assert np.allclose(gate[r, q], softmax(sel), rtol=0, atol=1e-14)
            assert abs(gate[r, q].sum() - 1.0) < 1e-14 and (gate[r, q] > 0).all()


# --------------------------------------------------------------------------
# Compaction
# --------------------------------------------------------------------------

def check_compact(o):
    """Packed lists equal np.nonzero of the selection mask; lists strictly
    increasing; every selected (t, j) appears once; totals are T*g*k."""
    B, T, h, g, k = 3, 37, 8, 2, 2
    x = _f32((B, T, 12), 31)
    W = _f32((12, h), 32)
    idx, _, _, _ = o.route(x, W, h, g, k)
    offs, pos = o.compact(idx, h, g, k)
    mask = np.zeros((B, T, h), bool)
    for b in range(B):
        for t in range(T):
            mask[b, t, idx[b, t].reshape(-1)] = True
    assert offs[0] == 0 and offs[-1] == B * T * g * k
    for b in range(B):
        for j in range(h):
            lst = pos[offs[b * h + j]:offs[b * h + j + 1]]
            assert np.array_equal(lst, np.nonzero(mask[b, :, j])[0]), "list != nonzero(mask)"
            assert (np.diff(lst) > 0).all()
        assert offs[(b + 1) * h] - offs[b * h] == T * g * k


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _random_routing(B, T, h, g, k, seed):
    """Random valid routing (k distinct heads of each group, positive gates
    summing to one), independent of the router."""
    r = _rng(seed)
    hpg = h // g
    idx = np.empty((B, T, g, k), np.int32)
    gate = np.empty((B, T, g, k), np.float64)
    for b in range(B):
        for t in range(T):
            for q in range(g):
                idx[b, t, q] = q * hpg + r.permutation(hpg)[:k]
                w = r.random(k) + 0.1
                gate[b, t, q] = w / w.sum()
    return idx, gate


def _sdpa_expected(Q, K, V, idx, gate):
    """gate * causal SDPA (torch, fp64, GQA expansion) for selected heads, 0 elsewhere."""
    q = torch.from_numpy(Q.astype(np.float64)).transpose(1, 2)
    kk = torch.from_numpy(K.astype(np.float64)).transpose(1, 2)
    vv = torch.from_numpy(V.astype(np.float64)).transpose(1, 2)
    full = F.scaled_dot_product_attention(q, kk, vv, is_causal=True, enable_gqa=True)
    full = full.transpose(1, 2).numpy()  # [B, T, h, d]
    B, T, h, d = Q.shape
    out = np.zeros_like(full)
    for b in range(B):
        for t in range(T):
            for q_ in range(idx.shape[2]):
                for s in range(idx.shape[3]):
                    j = idx[b, t, q_, s]
                    out[b, t, j] = gate[b, t, q_, s] * full[b, t, j]
    return out


def check_attn_sdpa(o):
    """Routed output = gate x torch SDPA(causal, GQA) on selected heads, zero elsewhere."""
    for (B, T, h, g, d, k, seed) in [(2, 19, 8, 2, 16, 2, 40), (1, 33, 6, 3, 8, 1, 41),
                                     (1, 12, 4, 1, 8, 4, 42), (1, 9, 4, 4, 8, 1, 43)]:
        Q = _f32((B, T, h, d), seed)
        K = _f32((B, T, g, d), seed + 1)
        V = _f32((B, T, g, d), seed + 2)
        idx, gate = _random_routing(B, T, h, g, k, seed + 3)
        got = o.attn(Q, K, V, idx, gate)
        want = _sdpa_expected(Q, K, V, idx, gate)
        assert np.abs(got - want).max() < 1e-12, f"SDPA mismatch {np.abs(got - want).max()}"


def check_attn_closed_forms(o):
    B, T, h, g, d, k = 1, 11, 4, 2, 8, 1
    idx, gate = _random_routing(B, T, h, g, k, 50)
    Q = _f32((B, T, h, d), 51)
    V = _f32((B, T, g, d), 52)
    # T = 1: the only visible key is the token itself -> O = gate * V[0]
    O1 = o.attn(Q[:, :1], _f32((B, 1, g, d), 53), V[:, :1], idx[:, :1], gate[:, :1])
    for q_ in range(g):
        j = idx[0, 0, q_, 0]
        assert np.allclose(O1[0, 0, j], gate[0, 0, q_, 0] * V[0, 0, q_].astype(np.float64), atol=1e-15)
    # K = 0: uniform weights over s <= t -> running mean of V
    O0 = o.attn(Q, np.zeros((B, T, g, d), np.float32), V, idx, gate)
    Vd = V.astype(np.float64)
    run_mean = np.cumsum(Vd, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    for t in range(T):
        for q_ in range(g):
            j = idx[0, t, q_, 0]
            assert np.allclose(O0[0, t, j], gate[0, t, q_, 0] * run_mean[0, t, q_], atol=1e-13)
    # constant V rows: output equals that row whatever the weights
    vc = _f32((g, d), 54)
    Vc = np.broadcast_to(vc, (B, T, g, d)).copy()
    Oc = o.attn(Q, _f32((B, T, g, d), 55), Vc, idx, gate)
    for t in range(T):
        for q_ in range(g):
            j = idx[0, t, q_, 0]
            assert np.allclose(Oc[0, t, j], gate[0, t, q_, 0] * vc[q_].astype(np.float64), atol=1e-13)
    # one dominant key at s* = 4: rows t >= 4 return V[s*], rows t < 4 see only zero scores
    Qd = np.zeros((B, T, h, d), np.float32)
    Qd[..., 0] = 30.0
    Kd = np.zeros((B, T, g, d), np.float32)
    Kd[0, 4, :, 0] = 30.0
    Od = o.attn(Qd, Kd, V, idx, gate)
    for t in range(T):
        for q_ in range(g):
            j = idx[0, t, q_, 0]
            want = Vd[0, 4, q_] if t >= 4 else run_mean[0, t, q_]
            assert np.allclose(Od[0, t, j], gate[0, t, q_, 0] * want, atol=1e-12), f"dominant key t={t}"


def check_mha_mqa(o):
    """g = h (MHA): one head per group, gate 1, output = causal SDPA without
    expansion.  g = 1 (MQA) with k = h: every head attends the single KV head."""
    B, T, h, d = 1, 14, 4, 8
    Q = _f32((B, T, h, d), 60)
    K = _f32((B, T, h, d), 61)
    V = _f32((B, T, h, d), 62)
    x = _f32((B, T, 5), 63)
    idx, gate, _, _ = o.route(x, _f32((5, h), 64), h, h, 1)
    assert (gate == 1.0).all()
    got = o.attn(Q, K, V, idx, gate)
    t = lambda a: torch.from_numpy(a.astype(np.float64)).transpose(1, 2)
    want = F.scaled_dot_product_attention(t(Q), t(K), t(V), is_causal=True).transpose(1, 2).numpy()
    assert np.abs(got - want).max() < 1e-12
    K1, V1 = K[:, :, :1], V[:, :, :1]
    idx, gate, _, _ = o.route(x, _f32((5, h), 65), h, 1, h)
    got = o.attn(Q, K1, V1, idx, gate)
    base = F.scaled_dot_product_attention(t(Q), t(K1).expand(B, h, T, d), t(V1).expand(B, h, T, d),
                                          is_causal=True).transpose(1, 2).numpy()
    g_of_head = np.zeros((B, T, h))
    for s in range(h):
        g_of_head[0, np.arange(T), idx[0, :, 0, s]] = gate[0, :, 0, s]
    assert np.abs(got - g_of_head[..., None] * base).max() < 1e-12


def check_prefix_invariance(o):
    """Truncating the sequence leaves the earlier rows bit-identical (causality)."""
    B, T, h, g, d, k = 2, 24, 8, 2, 16, 2
    Q = _f32((B, T, h, d), 70)
    K = _f32((B, T, g, d), 71)
    V = _f32((B, T, g, d), 72)
    idx, gate = _random_routing(B, T, h, g, k, 73)
    full = o.attn(Q, K, V, idx, gate)
    Tp = 13
    part = o.attn(Q[:, :Tp].copy(), K[:, :Tp].copy(), V[:, :Tp].copy(), idx[:, :Tp].copy(), gate[:, :Tp].copy())
    assert np.array_equal(full[:, :Tp], part)


def check_decode(o):
    """Decode of a query at position L-1 equals SDPA over cache rows 0..L-1, and
    equals the prefill row t = L-1 built from the same rows."""
    B, Lmax, h, g, d, k = 3, 21, 8, 2, 16, 2
    lengths = np.array([1, 13, 21], np.int32)
    q = _f32((B, 1, h, d), 80)
    Kc = _f32((B, Lmax, g, d), 81)
    Vc = _f32((B, Lmax, g, d), 82)
    idx, gate = _random_routing(B, 1, h, g, k, 83)
    got = o.decode(q, Kc, Vc, lengths, idx, gate)
    for b in range(B):
        L = int(lengths[b])
        qq = torch.from_numpy(q[b:b + 1].astype(np.float64)).transpose(1, 2)  # [1,h,1,d]
        kk = torch.from_numpy(Kc[b:b + 1, :L].astype(np.float64)).transpose(1, 2)
        vv = torch.from_numpy(Vc[b:b + 1, :L].astype(np.float64)).transpose(1, 2)
        full = F.scaled_dot_product_attention(qq, kk, vv, enable_gqa=True)[0, :, 0]  # [h, d]
        want = np.zeros((h, d))
        for q_ in range(g):
            for s in range(k):
                j = idx[b, 0, q_, s]
                want[j] = gate[b, 0, q_, s] * full[j].numpy()
        assert np.abs(got[b] - want).max() < 1e-12, f"decode b={b}"
        # decode <-> prefill: put q at position L-1 of a prefill over the cache rows
        Qp = np.zeros((1, L, h, d), np.float32)
        Qp[0, L - 1] = q[b, 0]
        ip = np.repeat(idx[b:b + 1], L, axis=1)
        gp = np.repeat(gate[b:b + 1], L, axis=1)
        row = o.attn_rows(Qp, Kc[b:b + 1, :L].copy(), Vc[b:b + 1, :L].copy(), ip, gp, rows=[L - 1])
        assert np.abs(row[0] - got[b]).max() < 1e-12


# --------------------------------------------------------------------------
# Worked examples printed on the pages (tests/golden)
# --------------------------------------------------------------------------

def check_group_map_golden(o):
    """freenetmedia.pl example: h=8, g=2 -> heads 0-3 use KV head 0, 4-7 KV head 1."""
    rows = read_golden("head_group_map.txt")
    h, g = rows[0][0], rows[0][1]
    expect = {r[0]: r[1] for r in rows[1:]}
    B, T, d = 1, 3, 4
    Q = _f32((B, T, h, d), 90)
    K = _f32((B, T, g, d), 91)
    V = np.zeros((B, T, g, d), np.float32)
    for q_ in range(g):
        V[:, :, q_, :] = float(q_ + 1)  # KV head q carries the constant value q + 1
    x = _f32((B, T, 6), 92)
    idx, gate, _, _ = o.route(x, _f32((6, h), 93), h, g, h // g)  # every head selected
    O = o.attn(Q, K, V, idx, gate)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                for s in range(h // g):
                    j = idx[b, t, q_, s]
                    kv = O[b, t, j, 0] / gate[b, t, q_, s] - 1.0
                    assert abs(kv - expect[j]) < 1e-12, f"head {j} read KV head {kv}, pages say {expect[j]}"


def check_active_heads_golden(o):
    """gist.science main configuration: 16 query heads, 8 KV groups, k=1 ->
    8 routed query-head computations per token (the always-on shared head is a
    separate, extra head and not part of the routed output)."""
    h, g, k, routed = read_golden("active_heads.txt")[0]
    B, T, d = 1, 10, 8
    x = _f32((B, T, 32), 95)
    idx, gate, _, _ = o.route(x, _f32((32, h), 96), h, g, k)
    O = o.attn(_f32((B, T, h, d), 97), _f32((B, T, g, d), 98), _f32((B, T, g, d), 99), idx, gate)
    nonzero = (np.abs(O).sum(axis=-1) > 0).sum(axis=-1)
    assert (nonzero == routed).all(), f"nonzero head slots per token {set(nonzero.ravel())} != {routed}"


# --------------------------------------------------------------------------
# Output construction: shared head and per-group slots
# --------------------------------------------------------------------------

def check_shared_head_closed_forms(o):
    """The shared head attends causally to the chosen KV group only."""
    B, T, g, d = 2, 7, 3, 8
    kv = 2  # not group 0: the other groups' V differ, so a wrong group fails
    Qs = _f32((B, T, d), 70)
    V = _f32((B, T, g, d), 71)
    Vd = V.astype(np.float64)
    # K = 0: uniform weights over s <= t -> running mean of the group's V
    Os = o.shared_rows(Qs, np.zeros((B, T, g, d), np.float32), V, kv).reshape(B, T, d)
    run_mean = np.cumsum(Vd[:, :, kv], axis=1) / np.arange(1, T + 1)[None, :, None]
    assert np.allclose(Os, run_mean, atol=1e-13), "shared head, K = 0"
    # T = 1: the token's own V row
    O1 = o.shared_rows(Qs[:, :1], _f32((B, 1, g, d), 72), V[:, :1], kv).reshape(B, d)
    assert np.allclose(O1, Vd[:, 0, kv], atol=1e-15), "shared head, T = 1"
    # one dominant key at s* = 3 in the chosen group: rows t >= 3 return V[s*]
    Qd = np.zeros((B, T, d), np.float32)
    Qd[..., 1] = 30.0
    Kd = np.zeros((B, T, g, d), np.float32)
    Kd[:, 3, kv, 1] = 30.0
    Od = o.shared_rows(Qd, Kd, V, kv).reshape(B, T, d)
    for t in range(T):
        want = Vd[:, 3, kv] if t >= 3 else run_mean[:, t]
        assert np.allclose(Od[:, t], want, atol=1e-12), f"shared head, dominant key t={t}"


def check_group_slots(o):
    """Each head's query dominates one key, so its attention output is exactly
    that key's V row (the other weights underflow to zero in double); the
    concatenated slots must follow the selection order and the weighted sum
    must pair each slot with its own gate."""
    B, T, h, g, d, k = 1, 4, 4, 2, 4, 2
    hpg = h // g
    key_of_head = [3, 1, 0, 2]
    K = np.zeros((B, T, g, d), np.float32)
    for s in range(T):
        K[0, s, :, s] = 40.0
    Q = np.zeros((B, T, h, d), np.float32)
    for j in range(h):
        Q[0, :, j, key_of_head[j]] = 40.0
    V = _f32((B, T, g, d), 73)
    Vd = V.astype(np.float64)
    idx = np.zeros((B, T, g, k), np.int32)
    gate = np.zeros((B, T, g, k), np.float64)
    for t in range(T):
        for q_ in range(g):
            order = [q_ * hpg + 1, q_ * hpg] if (t + q_) % 2 == 0 else [q_ * hpg, q_ * hpg + 1]
            idx[0, t, q_] = order
            gate[0, t, q_] = [0.7, 0.3] if t % 2 == 0 else [0.6, 0.4]
    t = T - 1  # every key visible
    cat, wsum = o.group_slots_rows(Q, K, V, idx, gate, rows=[t])
    for q_ in range(g):
        want_w = np.zeros(d)
        for r in range(k):
            j = idx[0, t, q_, r]
            want = Vd[0, key_of_head[j], q_]
            assert np.allclose(cat[0, q_, r], want, atol=1e-12), f"slot (q={q_}, r={r})"
            want_w += gate[0, t, q_, r] * want
        assert np.allclose(wsum[0, q_], want_w, atol=1e-12), f"weighted sum q={q_}"
    # T = 1: every selected head sees only its own token
    cat1, wsum1 = o.group_slots_rows(Q[:, :1], K[:, :1], V[:, :1], idx[:, :1], gate[:, :1], rows=[0])
    for q_ in range(g):
        assert np.allclose(cat1[0, q_], Vd[0, 0, q_][None, :], atol=1e-15)
        assert np.allclose(wsum1[0, q_], Vd[0, 0, q_] * gate[0, 0, q_].sum(), atol=1e-15)


# --------------------------------------------------------------------------
# Routed query projection
# --------------------------------------------------------------------------

def check_qproj(o):
    """Block-identity W_Q (d_model = h*d_h): each selected head's query row is
    exactly its own d_h-slice of x; a one-hot x picks one row of W_Q."""
    B, T, h, g, d, k = 2, 3, 4, 2, 4, 2
    d_model = h * d
    x = _f32((B, T, d_model), 80)
    idx = np.zeros((B, T, g, k), np.int32)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                idx[b, t, q_] = [q_ * 2 + 1, q_ * 2] if (b + t + q_) % 2 else [q_ * 2, q_ * 2 + 1]
    Wid = np.eye(d_model, dtype=np.float32)
    Qs = o.qproj_rows(x, Wid, idx, d).reshape(B, T, g, k, d)
    xd = x.astype(np.float64)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                for r in range(k):
                    j = idx[b, t, q_, r]
                    assert np.array_equal(Qs[b, t, q_, r], xd[b, t, j * d:(j + 1) * d]), f"identity W_Q ({b},{t},{q_},{r})"
    # one-hot x at input i: the query row of head j is row i of W_Q's j-th column block
    W = _f32((d_model, h * d), 81)
    i0 = 5
    x1 = np.zeros((B, T, d_model), np.float32)
    x1[:, :, i0] = 1.0
    Q1 = o.qproj_rows(x1, W, idx, d).reshape(B, T, g, k, d)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                for r in range(k):
                    j = idx[b, t, q_, r]
                    assert np.array_equal(Q1[b, t, q_, r], W[i0, j * d:(j + 1) * d].astype(np.float64))


# --------------------------------------------------------------------------
# Paged decode
# --------------------------------------------------------------------------

def check_decode_paged(o):
    """Pages in a permuted pool: zero keys give the mean of the sequence's first
    L logical rows; a dominant key at logical position s* returns exactly that
    row; and the result equals the contiguous decode of the gathered cache."""
    B, ps, nb, npages, h, g, d, k = 2, 4, 3, 8, 4, 2, 8, 1
    hpg = h // g
    bt = np.array([[5, 2, 7], [1, 6, 0]], np.int32)
    lengths = np.array([10, 5], np.int32)
    q = _f32((B, h, d), 90)
    Vp = _f32((npages, ps, g, d), 91)
    idx = np.array([[[0], [3]], [[1], [2]]], np.int32)  # [B, g, k]: one head per group
    gate = np.ones((B, g, k), np.float64)

    def logical(P, b, s_):
        return P[bt[b, s_ // ps], s_ % ps]

    Vd = Vp.astype(np.float64)
    # zero keys: uniform weights over the L logical rows
    O0 = o.decode_paged(q, np.zeros_like(Vp), Vp, bt, lengths, idx, gate)
    for b in range(B):
        mean = np.mean([logical(Vd, b, s_) for s_ in range(lengths[b])], axis=0)  # [g, d]
        for q_ in range(g):
            assert np.allclose(O0[b, idx[b, q_, 0]], mean[q_], atol=1e-13), f"paged K=0 b={b}"
    # dominant key at logical position s* (order-sensitive)
    star = [7, 3]
    Kp = np.zeros_like(Vp)
    qd = np.zeros_like(q)
    qd[..., 0] = 30.0
    for b in range(B):
        pg, r = bt[b, star[b] // ps], star[b] % ps
        Kp[pg, r, :, 0] = 30.0
    Od = o.decode_paged(qd, Kp, Vp, bt, lengths, idx, gate)
    for b in range(B):
        for q_ in range(g):
            assert np.allclose(Od[b, idx[b, q_, 0]], logical(Vd, b, star[b])[q_], atol=1e-12), f"paged s* b={b}"
    # the gathered cache through the contiguous decode
    Kp2 = _f32((npages, ps, g, d), 92)
    Lmax = ps * nb
    Kc = np.zeros((B, Lmax, g, d), np.float32)
    Vc = np.zeros((B, Lmax, g, d), np.float32)
    for b in range(B):
        for s_ in range(lengths[b]):
            Kc[b, s_] = logical(Kp2, b, s_)
            Vc[b, s_] = logical(Vp, b, s_)
    idx2 = np.array([[[1], [2]], [[0], [3]]], np.int32)
    gate2 = np.full((B, g, k), 0.75)
    Op = o.decode_paged(q, Kp2, Vp, bt, lengths, idx2, gate2)
    Oc = o.decode(q, Kc, Vc, lengths, idx2, gate2)
    # (the gate enters each weight here and the finished row there: agreement to rounding)
    assert np.allclose(Op, Oc, rtol=0, atol=1e-12), "paged decode differs from the contiguous decode of the gathered cache"
    for b in range(B):
        for j in range(h):
            if j not in idx2[b].reshape(-1):
                assert np.all(Op[b, j] == 0.0)
    _ = hpg


# --------------------------------------------------------------------------
# Backward (training)
# --------------------------------------------------------------------------

def _gate_mask(idx, gate, h):
    """[B, T, h] with gate_j in selected slots and 0 elsewhere."""
    B, T, g, k = idx.shape
    m = np.zeros((B, T, h))
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                for s in range(k):
                    m[b, t, idx[b, t, q_, s]] = gate[b, t, q_, s]
    return m


def check_backward_sdpa_autograd(o):
    """dQ, dK, dV, dgate = torch autograd (fp64) of sum(dO * mask * SDPA(causal, GQA)),
    mask = gate in selected slots, 0 elsewhere: a library routine's own backward."""
    for (B, T, h, g, d, k, seed) in [(2, 13, 8, 2, 8, 2, 600), (1, 17, 6, 3, 4, 1, 601), (1, 9, 4, 1, 8, 4, 602)]:
        Q = _f32((B, T, h, d), seed)
        K = _f32((B, T, g, d), seed + 1)
        V = _f32((B, T, g, d), seed + 2)
        idx, gate = _random_routing(B, T, h, g, k, seed + 3)
        dO = _rng(seed + 4).standard_normal((B, T, h, d))
        dQ, dK, dV, dgate = o.attn_backward(Q, K, V, idx, gate, dO)
        q = torch.from_numpy(Q.astype(np.float64)).transpose(1, 2).requires_grad_()
        kk = torch.from_numpy(K.astype(np.float64)).transpose(1, 2).requires_grad_()
        vv = torch.from_numpy(V.astype(np.float64)).transpose(1, 2).requires_grad_()
        full = F.scaled_dot_product_attention(q, kk, vv, is_causal=True, enable_gqa=True).transpose(1, 2)
        m = torch.from_numpy(_gate_mask(idx, gate, h))[..., None]
        (full * m * torch.from_numpy(dO)).sum().backward()
        for name, got, want in (("dQ", dQ, q.grad.transpose(1, 2)), ("dK", dK, kk.grad.transpose(1, 2)),
                                ("dV", dV, vv.grad.transpose(1, 2))):
            err = np.abs(got - want.numpy()).max()
            assert err < 1e-12, f"{name} vs autograd: {err}"
        fo = full.detach().numpy()
        for b in range(B):
            for t in range(T):
                for q_ in range(g):
                    for s in range(k):
                        j = idx[b, t, q_, s]
                        want = float(np.dot(dO[b, t, j], fo[b, t, j]))
                        assert abs(dgate[b, t, q_, s] - want) < 1e-12, "dgate vs SDPA output"


def _central(f, a, i, eps):
    """Central difference of f along element i of the fp32 array a, dividing by
    the step actually taken after rounding to fp32."""
    x0 = a.flat[i]
    ap, am = a.copy(), a.copy()
    ap.flat[i] = np.float32(x0 + eps)
    am.flat[i] = np.float32(x0 - eps)
    return (f(ap) - f(am)) / (float(ap.flat[i]) - float(am.flat[i]))


def check_backward_finite_differences(o):
    """Gradients of L = sum(dO * O) against central differences of the forward
    oracle, for Q, K, V, the gates, and (through the router) x, W_r and bias.
    Two routings: every head of a group selected (k = h/g), and 2 of 3."""
    for (B, T, h, g, d, k, d_model, seed) in [(1, 6, 4, 2, 4, 2, 5, 610), (1, 5, 6, 2, 4, 2, 5, 670)]:
        _fd_case(o, B, T, h, g, d, k, d_model, seed)


def _fd_case(o, B, T, h, g, d, k, d_model, seed):
    Q = _f32((B, T, h, d), seed)
    K = _f32((B, T, g, d), seed + 1)
    V = _f32((B, T, g, d), seed + 2)
    dO = _rng(seed + 3).standard_normal((B, T, h, d))
    x = _f32((B, T, d_model), seed + 4)
    W = _f32((d_model, h), seed + 5, 0.7)
    bias = _f32((h,), seed + 6, 0.3)
    idx, gate, _, margin = o.route(x, W, h, g, k, bias=bias)
    assert margin.min() > 0.05 or k == h // g, "test inputs must keep the selection away from ties"
    dQ, dK, dV, dgate = o.attn_backward(Q, K, V, idx, gate, dO)
    eps = 1e-3
    tol = 2e-6
    for name, arr, grad in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        def loss(a, name=name):
            args = {"Q": Q, "K": K, "V": V}
            args[name] = a
            return float((o.attn(args["Q"], args["K"], args["V"], idx, gate) * dO).sum())
        for i in range(arr.size):
            fd = _central(loss, arr, i, eps)
            assert abs(fd - grad.flat[i]) < tol * (1 + abs(fd)), f"d{name}[{i}]: fd {fd} vs {grad.flat[i]}"
    for i in range(gate.size):  # O is linear in each gate
        gp, gm = gate.copy(), gate.copy()
        gp.flat[i] += 0.5
        gm.flat[i] -= 0.5
        fd = float(((o.attn(Q, K, V, idx, gp) - o.attn(Q, K, V, idx, gm)) * dO).sum())
        assert abs(fd - dgate.flat[i]) < 1e-10 * (1 + abs(fd)), f"dgate[{i}]"
    dl, dx, dW, db = o.route_backward(x, W, idx, gate, dgate)

    def layer(xx, WW, bb):
        i2, g2, _, _ = o.route(xx, WW, h, g, k, bias=bb)
        assert np.array_equal(i2, idx), "a finite-difference step changed the selection"
        return float((o.attn(Q, K, V, i2, g2) * dO).sum())
    eps_r, tol_r = 1e-2, 2e-4  # the router's fp32 logits add rounding noise to each difference
    for name, arr, grad in (("x", x, dx), ("W_r", W, dW), ("bias", bias, db)):
        def loss(a, name=name):
            args = {"x": x, "W_r": W, "bias": bias}
            args[name] = a
            return layer(args["x"], args["W_r"], args["bias"])
        for i in range(arr.size):
            fd = _central(loss, arr, i, eps_r)
            assert abs(fd - grad.flat[i]) < tol_r * (1 + abs(fd)), f"d{name}[{i}]: fd {fd} vs {grad.flat[i]}"


def check_backward_invariants(o):
    """Softmax shift invariance: each attention row's score gradients sum to 0,
    so sum_s dK[b,s,q] = 0, and each group's logit gradients sum to 0.  Closed
    forms with K = 0 (uniform weights): dQ = 0 and
    dV[b,s,q] = sum_{t>=s} sum_{j in S(t,q)} gate_j dO[b,t,j] / (t+1).
    With one head per group (g = h) the gate is 1 and the logit gradient 0."""
    B, T, h, g, d, k = 2, 10, 6, 2, 8, 2
    Q = _f32((B, T, h, d), 620)
    K = _f32((B, T, g, d), 621)
    V = _f32((B, T, g, d), 622)
    idx, gate = _random_routing(B, T, h, g, k, 623)
    dO = _rng(624).standard_normal((B, T, h, d))
    dQ, dK, dV, dgate = o.attn_backward(Q, K, V, idx, gate, dO)
    assert np.abs(dK.sum(axis=1)).max() < 1e-12, "sum_s dK != 0"
    sel = _gate_mask(idx, gate, h) > 0
    assert np.all(dQ[~sel] == 0.0), "dQ of an unselected slot"
    x = _f32((B, T, 7), 625)
    W = _f32((7, h), 626)
    dl, _, _, _ = o.route_backward(x, W, idx, gate, dgate)
    assert np.abs(dl.reshape(B, T, g, h // g).sum(axis=-1)).max() < 1e-12, "sum of a group's dlogits != 0"
    assert np.all(dl[~sel] == 0.0), "dlogit of an unselected head"
    dQ0, _, dV0, dg0 = o.attn_backward(Q, np.zeros_like(K), V, idx, gate, dO)
    assert np.abs(dQ0).max() < 1e-13, "dQ with K = 0"
    want = np.zeros_like(dV0)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                for s in range(k):
                    j = idx[b, t, q_, s]
                    want[b, : t + 1, q_] += gate[b, t, q_, s] * dO[b, t, j] / (t + 1)
                    assert abs(dg0[b, t, q_, s] - np.dot(dO[b, t, j], V[b, : t + 1, q_].astype(np.float64).mean(0))) < 1e-12
    assert np.abs(dV0 - want).max() < 1e-12, "dV with K = 0"
    # a suffix of query rows: the later key rows of dK/dV and the later query rows are exact
    tq, tk, tv, tg = o.attn_backward(Q, K, V, idx, gate, dO, t_min=6)
    for name, got, want in (("dK", tk, dK), ("dV", tv, dV), ("dQ", tq, dQ), ("dgate", tg, dgate)):
        assert np.array_equal(got[:, 6:], want[:, 6:]), f"t_min: {name} rows past t_min"
    assert np.all(tq[:, :6] == 0.0) and np.all(tg[:, :6] == 0.0), "t_min: query rows before t_min"
    i1 = np.broadcast_to(np.arange(h, dtype=np.int32).reshape(1, 1, h, 1), (B, T, h, 1)).copy()
    g1 = np.ones((B, T, h, 1))
    _, _, _, dg1 = o.attn_backward(Q, np.repeat(K, 3, axis=2), np.repeat(V, 3, axis=2), i1, g1, dO)
    dl1, _, _, _ = o.route_backward(x, W, i1, g1, dg1)
    assert np.all(dl1 == 0.0), "one head per group: the logit gradient must be 0"


def check_aux_loss(o):
    """Load-balancing loss: equal logits give exactly 1 whatever the selection;
    a balanced routing (token t of each group favours head t, k = 1) gives 1
    and a zero gradient; a collapsed routing (every token on head 0 with
    probability ~1) gives h/g; the gradient matches central differences of the
    loss with the selection held fixed, and sums to 0 over each group."""
    N, h, g, k = 6, 6, 2, 2
    hpg = h // g
    idx = np.stack([np.stack([q * hpg + (np.arange(k) + t) % hpg for q in range(g)]) for t in range(N)]).astype(np.int32)
    L, dl = o.aux_loss(np.zeros((N, h), np.float32), idx)
    assert abs(L - 1.0) < 1e-15, f"equal logits: {L}"
    # balanced: N = hpg tokens, token t puts +2 on head t of every group, selects it (k = 1)
    lb = np.zeros((hpg, h), np.float32)
    ib = np.zeros((hpg, g, 1), np.int32)
    for t in range(hpg):
        for q in range(g):
            lb[t, q * hpg + t] = 2.0
            ib[t, q, 0] = q * hpg + t
    L, dl = o.aux_loss(lb, ib)
    assert abs(L - 1.0) < 1e-14 and np.abs(dl).max() < 1e-15, f"balanced: {L}, {np.abs(dl).max()}"
    # collapsed: head 0 of every group at +60, always selected
    lc = np.zeros((N, h), np.float32)
    lc[:, ::hpg] = 60.0
    ic = np.zeros((N, g, 1), np.int32)
    ic[:, :, 0] = np.arange(g) * hpg
    L, _ = o.aux_loss(lc, ic)
    assert abs(L - hpg) < 1e-12, f"collapsed: {L}"
    # gradient: central differences with the selection fixed, on a skewed
    # selection (head 0 of each group in every token's pair: f = 1/2, 1/4, 1/4)
    lr = _f32((N, h), 700)
    isk = np.stack([np.stack([q * hpg + np.array([0, 1 + t % 2]) for q in range(g)]) for t in range(N)])
    isk = isk.astype(np.int32)
    L0, dl = o.aux_loss(lr, isk)
    assert np.abs(dl).max() > 1e-3, "the skewed selection must give a gradient"
    assert np.abs(dl.reshape(N, g, hpg).sum(-1)).max() < 1e-15, "group sum of the gradient"
    for i in range(lr.size):
        fd = _central(lambda a: o.aux_loss(a, isk)[0], lr, i, 1e-3)
        assert abs(fd - dl.flat[i]) < 1e-7, f"aux dlogits[{i}]: fd {fd} vs {dl.flat[i]}"


# --------------------------------------------------------------------------
# Routed output projection
# --------------------------------------------------------------------------

def check_oproj(o):
    """Block-identity W_Z (d_model = h*d_h): a token's output is its selected
    heads' slots in place and zeros elsewhere, even where an unselected slot
    holds values (only the selected experts enter); a one-hot O at one
    element of a selected head returns that row of W_Z; with zeros in the
    unselected slots the result is the dense product of the concatenated
    heads with W_Z (numpy, fp64)."""
    B, T, h, g, d, k = 2, 3, 4, 2, 4, 1
    hpg = h // g
    idx = np.zeros((B, T, g, k), np.int32)
    for b in range(B):
        for t in range(T):
            for q_ in range(g):
                idx[b, t, q_, 0] = q_ * hpg + (b + 2 * t + q_) % hpg
    sel = np.zeros((B, T, h), bool)
    for b in range(B):
        for t in range(T):
            sel[b, t, idx[b, t].ravel()] = True
    O = _f32((B, T, h, d), 90)  # unselected slots deliberately non-zero
    Y = o.oproj_rows(O, np.eye(h * d, dtype=np.float32), idx).reshape(B, T, h, d)
    Od = O.astype(np.float64)
    for b in range(B):
        for t in range(T):
            for j in range(h):
                want = Od[b, t, j] if sel[b, t, j] else np.zeros(d)
                assert np.array_equal(Y[b, t, j], want), f"identity W_Z ({b},{t},{j})"
    # one-hot O at element c0 of token (1, 2)'s first selected head: that row of W_Z
    d_model = 7
    W = _f32((h * d, d_model), 91)
    c0 = 3
    O1 = np.zeros((B, T, h, d), np.float32)
    j0 = int(idx[1, 2, 1, 0])
    O1[1, 2, j0, c0] = 1.0
    Y1 = o.oproj_rows(O1, W, idx).reshape(B, T, d_model)
    assert np.array_equal(Y1[1, 2], W[j0 * d + c0].astype(np.float64)), "one-hot O picks a W_Z row"
    assert not Y1[0].any() and not Y1[1, :2].any()
    # zeros in the unselected slots: the dense product
    Oz = np.where(sel[..., None], O, 0.0).astype(np.float32)
    Yz = o.oproj_rows(Oz, W, idx).reshape(B, T, d_model)
    dense = Oz.reshape(B, T, h * d).astype(np.float64) @ W.astype(np.float64)
    assert np.allclose(Yz, dense, rtol=0, atol=1e-12), "dense product"


ALL_CHECKS = [
    check_router_onehot, check_router_bruteforce, check_router_zero_weights, check_gates,
    check_compact, check_attn_sdpa, check_attn_closed_forms, check_mha_mqa,
    check_prefix_invariance, check_decode, check_group_map_golden, check_active_heads_golden,
    check_shared_head_closed_forms, check_group_slots, check_qproj, check_decode_paged,
    check_backward_sdpa_autograd, check_backward_finite_differences, check_backward_invariants,
    check_aux_loss, check_oproj,
]
