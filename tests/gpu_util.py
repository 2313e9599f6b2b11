"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs, run the oracle on the same inputs, compare.

Comparison rules:
  * Routing: selections must match exactly, except for tokens whose oracle
    top-k logit margin l_(k) - l_(k+1) is below 1e-5 in some group (counted and
    returned).  Within a selection the order must follow the oracle's logits
    (descending) wherever adjacent logits differ by at least 1e-5.
  * Gates: within 1e-5 of the oracle's (fp32 exp vs double).
  * Outputs: max |O_gpu - O_oracle| <= 1e-4 (fp32) or 2e-2 (bf16) on every
    compared row; rows of excluded tokens are skipped.
"""
from __future__ import annotations

import numpy as np
import torch

import gqe_synth
import oracle
from routed_head_gqa_b200 import build as gqe_build

MARGIN_EXCLUDE = 1e-5
GATE_TOL = 1e-5
TOL = {"f32": 1e-4, "bf16": 2e-2}


def gqe():
    gqe_build.build()
    import routed_head_gqa_b200 as g

    return g


def to_dev(t, dev="cuda"):
    return None if t is None else t.to(dev)


def run_prefill(w, inp, dev="cuda"):
    """Route + prefill on the GPU.  Returns the Buffers (device tensors)."""
    g = gqe()
    shape = g.make_shape(w.B, w.T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, dev)
    buf.route(to_dev(inp["x"]), to_dev(inp["W_r"]), to_dev(inp["bias"]))
    buf.prefill(to_dev(inp["Q"]), to_dev(inp["K"]), to_dev(inp["V"]))
    torch.cuda.synchronize()
    st = buf.status()
    assert st == 0, f"device status {g.gqe_status_string(st)}"
    return buf


def run_decode(w, inp, dev="cuda"):
    g = gqe()
    shape = g.make_shape(w.B, 1, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
    buf = g.Buffers(shape, dev, Lmax=w.Lmax)
    buf.route(to_dev(inp["x"]), to_dev(inp["W_r"]), to_dev(inp["bias"]))
    buf.decode(to_dev(inp["q"]), to_dev(inp["K_cache"]), to_dev(inp["V_cache"]), to_dev(inp["lengths"]))
    torch.cuda.synchronize()
    st = buf.status()
    assert st == 0, f"device status {g.gqe_status_string(st)}"
    return buf


def oracle_route(w, inp):
    idx, gate, logits, margin = oracle.route(inp["x"], inp["W_r"], w.h, w.g, w.k, bias=inp["bias"])
    return idx, gate, logits, margin


def check_routing(w, inp, idx_gpu, gate_gpu):
    """Compare GPU routing with the oracle's.  Returns (excluded token mask [B, T],
    oracle idx, oracle gate)."""
    idx_o, gate_o, logits_o, margin_o = oracle_route(w, inp)
    idx_g = idx_gpu.cpu().numpy()
    gate_g = gate_gpu.cpu().numpy().astype(np.float64)
    excl = (margin_o < MARGIN_EXCLUDE).any(axis=-1)  # [B, T]
    keep = ~excl
    # selection sets and per-head gates, on kept tokens
    B, T, g_, k = idx_o.shape
    hot_o = np.zeros((B, T, w.h))
    hot_g = np.zeros((B, T, w.h))
    np.put_along_axis(hot_o, idx_o.reshape(B, T, -1), gate_o.reshape(B, T, -1), axis=-1)
    np.put_along_axis(hot_g, idx_g.reshape(B, T, -1), gate_g.reshape(B, T, -1), axis=-1)
    sel_o = np.zeros((B, T, w.h), bool)
    sel_g = np.zeros((B, T, w.h), bool)
    np.put_along_axis(sel_o, idx_o.reshape(B, T, -1), True, axis=-1)
    np.put_along_axis(sel_g, idx_g.reshape(B, T, -1), True, axis=-1)
    assert np.array_equal(sel_o[keep], sel_g[keep]), "routing selection differs from the oracle"
    assert np.abs(hot_o[keep] - hot_g[keep]).max(initial=0.0) < GATE_TOL, "gates differ from the oracle"
    # order inside each selection: descending oracle logit where distinguishable
    lg_sel = np.take_along_axis(logits_o.astype(np.float64).reshape(B, T, 1, -1).repeat(g_, 2),
                                idx_g.reshape(B, T, g_, k), axis=-1)
    if k > 1:
        gaps = lg_sel[..., :-1] - lg_sel[..., 1:]
        bad = (gaps < -MARGIN_EXCLUDE) & keep[..., None, None]
        assert not bad.any(), "selected heads not ordered by logit"
    # each token selects exactly k distinct heads of every group
    grp = idx_g // (w.h // w.g)
    assert (grp == np.arange(g_)[None, None, :, None]).all(), "selected head outside its group"
    return excl, idx_o, gate_o


def check_compaction(w, idx_gpu, offs_gpu, pos_gpu, chunk_gpu, excl, idx_o):
    """Packed lists: valid for the GPU's own selection (any size), and equal to
    the oracle's lists wherever the routing is not excluded."""
    B, T, h = w.B, w.T, w.h
    idx_g = idx_gpu.cpu().numpy()
    offs = offs_gpu.cpu().numpy()
    pos = pos_gpu.cpu().numpy()
    chunk = chunk_gpu.cpu().numpy().reshape(B, h, -1)
    nchunk = chunk.shape[-1]
    assert offs[0] == 0 and offs[-1] == B * T * w.g * w.k
    sel_g = np.zeros((B, T, h), bool)
    np.put_along_axis(sel_g, idx_g.reshape(B, T, -1), True, axis=-1)
    for b in range(B):
        for j in range(h):
            lst = pos[offs[b * h + j]:offs[b * h + j + 1]]
            assert np.array_equal(lst, np.nonzero(sel_g[b, :, j])[0]), f"list (b={b}, j={j}) invalid"
            # chunk offsets: first entry with t >= 32c
            want = offs[b * h + j] + np.searchsorted(lst, 32 * np.arange(nchunk))
            assert np.array_equal(chunk[b, j], want), f"chunk offsets (b={b}, j={j}) invalid"
    if not excl.any():
        offs_o, pos_o = oracle.compact(idx_o, w.h, w.g, w.k)
        assert np.array_equal(offs, offs_o) and np.array_equal(pos, pos_o), "lists differ from the oracle's"


def compare_rows(w, inp, O_gpu, idx_o, gate_o, excl, rows=None):
    """Oracle rows (b*T + t) vs the GPU output.  Returns (max error, rows compared)."""
    B, T = w.B, w.T
    if rows is None:
        rows = np.arange(B * T)
    rows = np.asarray(rows, dtype=np.int64)
    rows = rows[~excl.reshape(-1)[rows]]
    want = oracle.attn_rows(inp["Q"], inp["K"], inp["V"], idx_o, gate_o, rows=rows)
    got = O_gpu.float().reshape(B * T, w.h, w.d_h)[torch.from_numpy(rows).to(O_gpu.device)].cpu().numpy()
    err = float(np.abs(got.astype(np.float64) - want).max(initial=0.0))
    return err, len(rows)


def sm_count(dev=0):
    return torch.cuda.get_device_properties(dev).multi_processor_count


def prefill_windows(w):
    """(W, number of 2W-position windows) of the tensor-core prefill's work
    units: a unit is (b, KV group, window of 2W positions), W = 32*floor(4/k)."""
    W = 32 * (4 // w.k)
    return W, -(-w.T // (2 * W))


def cta_units(w, sms, cta):
    """The (b, q, window) units that CTA `cta` of the persistent prefill grid
    runs, in its order: unit j of CTA c is j*grid + (c, or grid-1-c for odd j),
    units ordered heaviest window first with (b, q) fastest."""
    _, nwin = prefill_windows(w)
    n_units = w.B * w.g * nwin
    grid = min(n_units, sms)
    out = []
    j = 0
    while True:
        unit = j * grid + ((grid - 1 - cta) if (j & 1) else cta)
        if unit >= n_units:
            break
        wr, rem = divmod(unit, w.B * w.g)
        out.append((rem // w.g, rem % w.g, nwin - 1 - wr))
        j += 1
    return out


def cover_rows(w, idx_o, sms, n_min=4096, seed=4321):
    """Flattened rows (b*T + t) for a full-size parity check that reaches
    every path of the persistent prefill: every position of the first, a middle
    and the last unit run by the first, a middle and the last CTA (first units
    exercise the pipeline fill, later ones the double-buffered row tables,
    barrier phases and TMEM reuse across units), every sequence's last window,
    the three windows with the most skewed head loads, then seeded random rows
    up to n_min.  Whole windows are compared for every head."""
    W, nwin = prefill_windows(w)
    span = 2 * W
    wins = set()
    grid = min(w.B * w.g * nwin, sms)
    for c in sorted({0, grid // 2, grid - 1}):
        units = cta_units(w, sms, c)
        for j in sorted({0, len(units) // 2, len(units) - 1}):
            b, _, win = units[j]
            wins.add((b, win))
    wins |= {(b, nwin - 1) for b in range(w.B)}
    # skew: the largest share of one head among a window's routed rows of one group
    sel = np.zeros((w.B, w.T, w.h), bool)
    np.put_along_axis(sel, idx_o.reshape(w.B, w.T, -1).astype(np.int64), True, axis=-1)
    pad = nwin * span - w.T
    per = np.pad(sel, ((0, 0), (0, pad), (0, 0))).reshape(w.B, nwin, span, w.h).sum(axis=2)
    skew = per.max(axis=-1)  # [B, nwin]
    for flat in np.argsort(-skew.reshape(-1), kind="stable")[:3]:
        wins.add((int(flat // nwin), int(flat % nwin)))
    rows = set()
    for b, win in wins:
        t0 = win * span
        rows.update(range(b * w.T + t0, b * w.T + min(t0 + span, w.T)))
    if len(rows) < n_min:
        gen = np.random.default_rng(seed)
        extra = gen.permutation(w.B * w.T)
        for r in extra:
            if len(rows) >= n_min:
                break
            rows.add(int(r))
    return np.array(sorted(rows), dtype=np.int64)


def prefill_parity(w, rows=None, cover=False):
    """Route + prefill on the GPU against the oracle.  rows: flattened rows to
    compare (all when None); cover=True picks them with cover_rows."""
    inp = gqe_synth.make_inputs(w)
    buf = run_prefill(w, inp)
    excl, idx_o, gate_o = check_routing(w, inp, buf.idx, buf.gate)
    check_compaction(w, buf.idx, buf.head_offsets, buf.head_pos, buf.head_chunk_offsets, excl, idx_o)
    if cover:
        rows = cover_rows(w, idx_o, sm_count())
    err, n = compare_rows(w, inp, buf.O, idx_o, gate_o, excl, rows)
    return err, n, int(excl.sum())


def decode_parity(w):
    inp = gqe_synth.make_inputs(w)
    buf = run_decode(w, inp)
    excl, idx_o, gate_o = check_routing(w, inp, buf.idx, buf.gate)
    want = oracle.decode(inp["q"], inp["K_cache"], inp["V_cache"], inp["lengths"], idx_o, gate_o)
    got = buf.O.float().reshape(w.B, w.h, w.d_h).cpu().numpy().astype(np.float64)
    keep = ~excl.reshape(-1)
    err = float(np.abs(got[keep] - want[keep]).max(initial=0.0))
    return err, int(keep.sum()), int(excl.sum())


def oracle_tables(w, idx_o, dev="cuda"):
    """Routing tables of the oracle's selection, for feeding the oracle's
    routing to a GPU kernel: (idx int32, head_offsets, head_pos,
    head_chunk_offsets) device tensors, the lists from oracle.compact and the
    per-32-position chunk starts found by search in each ascending list."""
    offs, pos = oracle.compact(idx_o, w.h, w.g, w.k)
    nchunk = (w.T + 31) // 32
    chunk = np.empty(w.B * w.h * nchunk, np.int32)
    for bj in range(w.B * w.h):
        lst = pos[offs[bj]:offs[bj + 1]]
        chunk[bj * nchunk:(bj + 1) * nchunk] = offs[bj] + np.searchsorted(lst, 32 * np.arange(nchunk), side="left")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    return t(idx_o), t(offs), t(pos), t(chunk)
