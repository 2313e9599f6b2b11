"""Seeded synthetic inputs for the GQE attention forward pass.

This module is the one thing the CUDA path and the CPU oracle share: it draws
input tensors and nothing else (no routing, no attention, no reductions).

Workloads (sizes, distributions and skews of the GQE prefill/decode cases):

  tiny_f32      B=1  T=128  d_model=256  h=8  g=2 d_h=32  k=1  fp32,
                W_r std 0.02
  dense_gqa     B=4  T=2048 d_model=4096 h=32 g=8 d_h=128 k=4  bf16,
                W_r std 1/64 (every head of every group selected: dense GQA
                up to the gates)
  gqe_prefill   B=8  T=4096 d_model=4096 h=32 g=8 d_h=128 k=2  bf16,
                W_r std 1/64 (near-uniform head loads)
  gqe_long      B=2  T=8192 d_model=2048 h=16 g=8 d_h=128 k=1  bf16,
                W_r std 1/sqrt(2048), +1.0 logit bias on head 0 of each group
                (skewed per-head token counts, about 76 % / 24 %)
  gqe_decode    B=64 one query token, cache lengths uniform in [1024, 16384],
                Lmax=16384, h=32 g=8 d_h=128 d_model=4096 k=2 bf16,
                W_r std 1/64, caches [B, Lmax, g, d_h]
  gqe_32k       B=1  T=32768 d_model=2048 h=16 g=8 d_h=128 k=1 bf16,
                W_r std 1/sqrt(2048) (a long-context case beyond the five)

Recipe: one CPU ``torch.Generator`` seeded with the workload's seed draws, in
this order, lengths (decode only), x, W_r, Q, K, V as fp32 standard normals
(W_r scaled by its std), then rounds bf16 workloads to bf16.  Decode caches are
drawn per sequence for rows 0 .. L_b-1 only; rows at or beyond L_b are zero and
are never read by the method.  The same values feed the GPU and the oracle.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    d_model: int
    h: int
    g: int
    d_h: int
    k: int
    dtype: str  # "f32" | "bf16"
    wr_std: float
    head0_bias: float = 0.0  # added to the logit of head 0 of every group
    decode: bool = False
    Lmin: int = 0
    Lmax: int = 0
    seed: int = 0

    @property
    def hpg(self) -> int:
        return self.h // self.g

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> str:
        s = (f"B={self.B} T={self.T} d_model={self.d_model} h={self.h} g={self.g} "
             f"d_h={self.d_h} k={self.k} {self.dtype}")
        if self.decode:
            s = (f"decode B={self.B} L~U[{self.Lmin},{self.Lmax}] d_model={self.d_model} "
                 f"h={self.h} g={self.g} d_h={self.d_h} k={self.k} {self.dtype}")
        return s


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 128, 256, 8, 2, 32, 1, "f32", 0.02, seed=0),
    "dense_gqa": Workload("dense_gqa", 4, 2048, 4096, 32, 8, 128, 4, "bf16", 1.0 / 64, seed=1),
    "gqe_prefill": Workload("gqe_prefill", 8, 4096, 4096, 32, 8, 128, 2, "bf16", 1.0 / 64, seed=2),
    "gqe_long": Workload("gqe_long", 2, 8192, 2048, 16, 8, 128, 1, "bf16", 1.0 / math.sqrt(2048),
                         head0_bias=1.0, seed=3),
    "gqe_decode": Workload("gqe_decode", 64, 1, 4096, 32, 8, 128, 2, "bf16", 1.0 / 64, decode=True,
                           Lmin=1024, Lmax=16384, seed=4),
    # Beyond the five configs: a 32k-token prefill with the GQE summary's main head
    # layout (16 query heads, 8 KV groups, k = 1), near-uniform router.
    "gqe_32k": Workload("gqe_32k", 1, 32768, 2048, 16, 8, 128, 1, "bf16", 1.0 / math.sqrt(2048), seed=5),
}


def custom(name="custom", *, B, T, d_model, h, g, d_h, k, dtype="bf16", wr_std=None,
           head0_bias=0.0, decode=False, Lmin=0, Lmax=0, seed=0) -> Workload:
    """A workload of any shape, with the same recipe (for parity tests)."""
    if wr_std is None:
        wr_std = 1.0 / math.sqrt(d_model)
    return Workload(name, B, T, d_model, h, g, d_h, k, dtype, wr_std, head0_bias, decode,
                    Lmin, Lmax, seed)


def _normal(shape, gen, std=1.0, chunk=1 << 25):
    """fp32 normals drawn in fixed-size chunks (deterministic for a given shape)."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = torch.randn(e - s, generator=gen)
    if std != 1.0:
        out.mul_(std)
    return out.view(*shape)


def bias_vector(w: Workload):
    """Per-head logit bias of the workload, or None (float32 [h])."""
    if w.head0_bias == 0.0:
        return None
    b = torch.zeros(w.h, dtype=torch.float32)
    b[:: w.hpg] = w.head0_bias
    return b


def make_inputs(w: Workload):
    """Draw the workload's inputs on the CPU.  Returns a dict of CPU tensors.

    prefill: x [B,T,d_model], W_r [d_model,h], Q [B,T,h,d_h], K/V [B,T,g,d_h], bias
    decode:  lengths [B] int32, x [B,1,d_model], W_r, q [B,1,h,d_h],
             K_cache/V_cache [B,Lmax,g,d_h], bias
    """
    gen = torch.Generator().manual_seed(w.seed)
    dt = w.torch_dtype
    out = {}
    if w.decode:
        lengths = torch.randint(w.Lmin, w.Lmax + 1, (w.B,), generator=gen, dtype=torch.int64)
        out["lengths"] = lengths.to(torch.int32)
        out["x"] = _normal((w.B, 1, w.d_model), gen).to(dt)
        out["W_r"] = _normal((w.d_model, w.h), gen, w.wr_std).to(dt)
        out["q"] = _normal((w.B, 1, w.h, w.d_h), gen).to(dt)
        for name in ("K_cache", "V_cache"):
            cache = torch.zeros((w.B, w.Lmax, w.g, w.d_h), dtype=dt)
            for b in range(w.B):
                L = int(lengths[b])
                cache[b, :L] = _normal((L, w.g, w.d_h), gen).to(dt)
            out[name] = cache
    else:
        out["x"] = _normal((w.B, w.T, w.d_model), gen).to(dt)
        out["W_r"] = _normal((w.d_model, w.h), gen, w.wr_std).to(dt)
        out["Q"] = _normal((w.B, w.T, w.h, w.d_h), gen).to(dt)
        out["K"] = _normal((w.B, w.T, w.g, w.d_h), gen).to(dt)
        out["V"] = _normal((w.B, w.T, w.g, w.d_h), gen).to(dt)
    out["bias"] = bias_vector(w)
    return out


def make_shared_query(w: Workload):
    """Query rows of the always-active shared head, Qs [B, T, d_h]: N(0, 1) in
    the workload's dtype, from their own seeded generator (seed + 7919), so the
    other inputs are unchanged."""
    gen = torch.Generator().manual_seed(w.seed + 7919)
    return _normal((w.B, w.T, w.d_h), gen).to(w.torch_dtype)


def make_paged_cache(K_cache, V_cache, page_size: int, seed: int = 4242, spare_pages: int = 3):
    """Cut contiguous caches [B, Lmax, g, d_h] into pages of page_size rows and
    scatter them over a pool in a seeded random order (plus a few unused
    pages).  Returns (K_pages, V_pages [num_pages, page_size, g, d_h],
    block_table int32 [B, max_blocks]) such that logical row s of sequence b is
    row s % page_size of page block_table[b, s // page_size]."""
    B, Lmax, g, d_h = K_cache.shape
    if Lmax % page_size:
        raise ValueError("Lmax must be a multiple of page_size")
    nb = Lmax // page_size
    num_pages = B * nb + spare_pages
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed))[: B * nb]
    K_pages = torch.zeros((num_pages, page_size, g, d_h), dtype=K_cache.dtype)
    V_pages = torch.zeros((num_pages, page_size, g, d_h), dtype=V_cache.dtype)
    K_pages[perm] = K_cache.reshape(B * nb, page_size, g, d_h)
    V_pages[perm] = V_cache.reshape(B * nb, page_size, g, d_h)
    return K_pages, V_pages, perm.to(torch.int32).reshape(B, nb)


def make_qproj_weight(w: Workload):
    """Query projection W_Q [d_model, h*d_h] ~ N(0, 1/sqrt(d_model)) in the
    workload's dtype (query rows of unit scale), from its own seeded generator
    (seed + 104729)."""
    gen = torch.Generator().manual_seed(w.seed + 104729)
    return _normal((w.d_model, w.h * w.d_h), gen, std=1.0 / math.sqrt(w.d_model)).to(w.torch_dtype)


def make_oproj_weight(w: Workload):
    """Output projection W_Z [h*d_h, d_model] ~ N(0, 1/sqrt(h*d_h)) in the
    workload's dtype, from its own seeded generator (seed + 130363)."""
    gen = torch.Generator().manual_seed(w.seed + 130363)
    return _normal((w.h * w.d_h, w.d_model), gen, std=1.0 / math.sqrt(w.h * w.d_h)).to(w.torch_dtype)


def make_random_routing(w: Workload, seed: int = 777, first_tile_fixed: bool = False):
    """A seeded routing with the router's structure but no router: for every
    (b, t, group q) k distinct heads of the group, drawn uniformly, as
    idx int32 [B, T, g, k].  first_tile_fixed: the first 128 tokens all take
    the group's first k heads (so a 128-token tile leaves heads unselected)."""
    gen = torch.Generator().manual_seed(w.seed + seed)
    hpg = w.h // w.g
    keys = torch.rand((w.B * w.T, w.g, hpg), generator=gen)
    pick = keys.argsort(dim=-1)[..., : w.k]
    if first_tile_fixed:
        pick[:128] = torch.arange(w.k)
    idx = pick + (torch.arange(w.g) * hpg)[None, :, None]
    return idx.to(torch.int32).reshape(w.B, w.T, w.g, w.k)


def make_routed_output(w: Workload, idx, seed: int = 991):
    """A stand-in for the gated routed output O [B, T, h, d_h]: N(0, 1/2) in
    the slots idx selects and exactly zero in every other slot (the layout the
    routed prefill writes), in the workload's dtype, from its own seeded
    generator."""
    gen = torch.Generator().manual_seed(w.seed + seed)
    O = _normal((w.B, w.T, w.h, w.d_h), gen, std=0.5)
    sel = torch.zeros((w.B * w.T, w.h), dtype=torch.bool)
    sel.scatter_(1, torch.as_tensor(idx).reshape(w.B * w.T, -1).long(), True)
    O[~sel.reshape(w.B, w.T, w.h)] = 0.0
    return O.to(w.torch_dtype)


def make_output_grad(w: Workload):
    """Incoming gradient dO [B,T,h,d_h] ~ N(0,1) in the workload's dtype (a
    stand-in for the gradient a training step would bring back), from its own
    seeded generator (seed + 31337)."""
    gen = torch.Generator().manual_seed(w.seed + 31337)
    return _normal((w.B, w.T, w.h, w.d_h), gen).to(w.torch_dtype)


def sample_rows(w: Workload, n: int, seed: int = 1234):
    """A seeded sample of n flattened token rows (b*T + t) that always includes
    the last position of every sequence and the first position of batch 0."""
    gen = torch.Generator().manual_seed(seed)
    total = w.B * w.T
    n = min(n, total)
    must = {0} | {b * w.T + w.T - 1 for b in range(w.B)}
    picks = torch.randperm(total, generator=gen)[: max(0, n - len(must))].tolist()
    rows = sorted(must | set(picks))
    return torch.tensor(rows, dtype=torch.int64)
