"""CPU oracle for the GQE attention forward pass -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use this package.  The product library (``routed_head_gqa_b200``)
never imports it, and it never imports the product library.

The arithmetic lives in ``gqe_oracle.c`` (plain C, double accumulation).  This
module only compiles it and marshals numpy arrays.  bf16 inputs are passed as
their raw 16-bit patterns (``uint16`` arrays); fp32 inputs as ``float32``.

Sources, per function (the same citations are in ``gqe_oracle.c``):
  route    -- "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
              (gist.science), "Architecture et Routage": top-k query-head
              experts per GQA group, renormalised router probabilities.
  compact  -- the per-(batch, head) packed position lists that the routed
              kernels consume (bookkeeping of the selection made by ``route``).
  attn_backward, route_backward -- the chain rule through the forward's own
              steps (attention, gating, renormalised gates, linear router).
  aux_loss -- the same page, "Entrainement et Perte": a load-balancing loss
              that spreads tokens evenly over each group's experts (read as
              the fraction-times-probability form; the page gives no formula).
  attn_rows, decode -- IBM "Que es la atencion de consultas agrupadas"
              (scaled dot-product attention, 1/sqrt(d_k)), ml-canon "56 GQA /
              MQA" (KV head expansion), freenetmedia.pl "Grouped-Query
              Attention" (contiguous head -> group mapping).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gqe_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1


def compile_source(src: str, out: str, strict: bool = True) -> str:
    """Compile an oracle C source file into a shared library (gcc, OpenMP).
    ``strict`` turns warnings into errors."""
    tmp = out + f".tmp{os.getpid()}"
    flags = ["-Wall", "-Werror"] if strict else []
    subprocess.check_call(["gcc", "-O2", *flags, "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile gqe_oracle.c into liboracle.so next to it (if stale)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, LIB_PATH)
    return LIB_PATH


def _as_input(a):
    """Return (contiguous numpy array, dtype code) for an fp32 or bf16 input.

    Accepts numpy float32 / uint16 arrays or CPU torch tensors (float32 or
    bfloat16); bf16 is handed over as its raw bit pattern."""
    if hasattr(a, "detach"):  # torch tensor
        import torch

        t = a.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), BF16
        if t.dtype == torch.float32:
            return t.numpy(), F32
        raise TypeError(f"oracle input dtype {t.dtype} not supported")
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle input dtype {a.dtype} not supported")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


class Oracle:
    """The oracle functions bound to one compiled library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        lib.oracle_route.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, P]
        lib.oracle_compact.argtypes = [i32, i32, i32, i32, i32, P, P, P]
        lib.oracle_attn_rows.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i64, P, P, i32]
        lib.oracle_decode.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i32]
        lib.oracle_shared_rows.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P, i32]
        lib.oracle_group_slots_rows.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i64, P, P, P,
                                                i32]
        lib.oracle_qproj_rows.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P, i32]
        lib.oracle_oproj_rows.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P, i32]
        lib.oracle_decode_paged.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i32]
        lib.oracle_attn_backward.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P,
                                             i32]
        lib.oracle_route_backward.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, i32]
        lib.oracle_aux_loss.argtypes = [i64, i32, i32, i32, P, P, P, P]
        for f in (lib.oracle_aux_loss, lib.oracle_route, lib.oracle_compact, lib.oracle_attn_rows, lib.oracle_decode,
                  lib.oracle_shared_rows, lib.oracle_group_slots_rows, lib.oracle_qproj_rows, lib.oracle_oproj_rows,
                  lib.oracle_decode_paged, lib.oracle_attn_backward, lib.oracle_route_backward):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = lib_path

    def route(self, x, W_r, h: int, g: int, k: int, bias=None):
        """Router: returns (idx int32 [..., g, k], gate float64 [..., g, k],
        logits float32 [..., h], margin float64 [..., g]) for x [..., d_model]."""
        xa, dt = _as_input(x)
        wa, dt2 = _as_input(W_r)
        if dt != dt2:
            raise TypeError("x and W_r must share a dtype")
        lead = xa.shape[:-1]
        d_model = xa.shape[-1]
        if wa.shape != (d_model, h):
            raise ValueError(f"W_r must be [{d_model}, {h}]")
        BT = int(np.prod(lead)) if lead else 1
        ba = None
        if bias is not None:
            ba = np.ascontiguousarray(np.asarray(bias, dtype=np.float32).reshape(h))
        logits = np.empty(lead + (h,), np.float32)
        idx = np.empty(lead + (g, k), np.int32)
        gate = np.empty(lead + (g, k), np.float64)
        margin = np.empty(lead + (g,), np.float64)
        rc = self.lib.oracle_route(BT, d_model, h, g, k, dt, _ptr(xa), _ptr(wa), _ptr(ba),
                                   _ptr(logits), _ptr(idx), _ptr(gate), _ptr(margin))
        if rc:
            raise ValueError(f"oracle_route failed ({rc})")
        return idx, gate, logits, margin

    def compact(self, idx, h: int, g: int, k: int):
        """Per-(batch, head) ascending position lists:
        (head_offsets int32 [B*h+1], head_pos int32 [B*T*g*k]) for idx [B, T, g, k]."""
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        B, T = ia.shape[0], ia.shape[1]
        offs = np.empty(B * h + 1, np.int32)
        pos = np.empty(B * T * g * k, np.int32)
        rc = self.lib.oracle_compact(B, T, h, g, k, _ptr(ia), _ptr(offs), _ptr(pos))
        if rc:
            raise ValueError(f"oracle_compact failed ({rc})")
        return offs, pos

    def attn_rows(self, Q, K, V, idx, gate, rows=None, n_threads=None):
        """GQE output rows O[b, t, :, :] (float64 [n_rows, h, d_h]) for the
        flattened token indices ``rows`` (b*T + t); all rows when None."""
        qa, dt = _as_input(Q)
        ka, dk = _as_input(K)
        va, dv = _as_input(V)
        if not (dt == dk == dv):
            raise TypeError("Q, K, V must share a dtype")
        B, T, h, d_h = qa.shape
        g = ka.shape[2]
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        ga = np.ascontiguousarray(gate, dtype=np.float64)
        k = ia.shape[-1]
        if rows is None:
            rows = np.arange(B * T, dtype=np.int64)
        ra = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
        out = np.empty((ra.shape[0], h, d_h), np.float64)
        rc = self.lib.oracle_attn_rows(B, T, h, g, d_h, k, dt, _ptr(qa), _ptr(ka), _ptr(va),
                                       _ptr(ia), _ptr(ga), ra.shape[0], _ptr(ra), _ptr(out),
                                       _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_attn_rows failed ({rc})")
        return out

    def shared_rows(self, Qs, K, V, kv_group: int, rows=None, n_threads=None):
        """Shared-head output (float64 [n_rows, d_h]) for Qs [B, T, d_h] (or
        [B, T, 1, d_h]) attending causally to KV group kv_group of K/V [B, T, g, d_h]."""
        qa, dt = _as_input(Qs)
        ka, dk = _as_input(K)
        va, dv = _as_input(V)
        if not (dt == dk == dv):
            raise TypeError("Qs, K, V must share a dtype")
        B, T, g, d_h = ka.shape
        qa = qa.reshape(B, T, d_h)
        if rows is None:
            rows = np.arange(B * T, dtype=np.int64)
        ra = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
        out = np.empty((ra.shape[0], d_h), np.float64)
        rc = self.lib.oracle_shared_rows(B, T, g, d_h, dt, int(kv_group), _ptr(qa), _ptr(ka), _ptr(va),
                                         ra.shape[0], _ptr(ra), _ptr(out), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_shared_rows failed ({rc})")
        return out

    def group_slots_rows(self, Q, K, V, idx, gate, rows=None, n_threads=None):
        """Per-group output slots for token rows b*T + t: (cat float64
        [n_rows, g, k, d_h], the selected heads' ungated outputs in selection
        order; wsum float64 [n_rows, g, d_h], their gate-weighted sum)."""
        qa, dt = _as_input(Q)
        ka, dk = _as_input(K)
        va, dv = _as_input(V)
        if not (dt == dk == dv):
            raise TypeError("Q, K, V must share a dtype")
        B, T, h, d_h = qa.shape
        g = ka.shape[2]
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        ga = np.ascontiguousarray(gate, dtype=np.float64)
        k = ia.shape[-1]
        if rows is None:
            rows = np.arange(B * T, dtype=np.int64)
        ra = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
        cat = np.empty((ra.shape[0], g, k, d_h), np.float64)
        wsum = np.empty((ra.shape[0], g, d_h), np.float64)
        rc = self.lib.oracle_group_slots_rows(B, T, h, g, d_h, k, dt, _ptr(qa), _ptr(ka), _ptr(va), _ptr(ia),
                                              _ptr(ga), ra.shape[0], _ptr(ra), _ptr(cat), _ptr(wsum),
                                              _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_group_slots_rows failed ({rc})")
        return cat, wsum

    def qproj_rows(self, x, W_Q, idx, d_h: int, rows=None, n_threads=None):
        """Routed query projection (float64 [n_rows, g, k, d_h]): the query row of
        each selected head idx[b,t,q,r] for token rows b*T + t."""
        xa, dt = _as_input(x)
        wa, dw = _as_input(W_Q)
        if dt != dw:
            raise TypeError("x and W_Q must share a dtype")
        B, T, d_model = xa.shape
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        g, k = ia.shape[2], ia.shape[3]
        h = wa.shape[1] // d_h
        if wa.shape != (d_model, h * d_h):
            raise ValueError("W_Q must be [d_model, h*d_h]")
        if rows is None:
            rows = np.arange(B * T, dtype=np.int64)
        ra = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
        out = np.empty((ra.shape[0], g, k, d_h), np.float64)
        rc = self.lib.oracle_qproj_rows(B, T, d_model, h, g, d_h, k, dt, _ptr(xa), _ptr(wa), _ptr(ia),
                                        ra.shape[0], _ptr(ra), _ptr(out), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_qproj_rows failed ({rc})")
        return out

    def oproj_rows(self, O, W_Z, idx, rows=None, n_threads=None):
        """Routed output projection (float64 [n_rows, d_model]) of token rows
        b*T + t: the sum over the token's selected heads j = idx[b,t,q,r] of
        O[b,t,j,:] . W_Z[j*d_h:(j+1)*d_h, :]."""
        oa, dt = _as_input(O)
        wa, dw = _as_input(W_Z)
        if dt != dw:
            raise TypeError("O and W_Z must share a dtype")
        B, T, h, d_h = oa.shape
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        g, k = ia.shape[2], ia.shape[3]
        if wa.ndim != 2 or wa.shape[0] != h * d_h:
            raise ValueError("W_Z must be [h*d_h, d_model]")
        d_model = wa.shape[1]
        if rows is None:
            rows = np.arange(B * T, dtype=np.int64)
        ra = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
        out = np.empty((ra.shape[0], d_model), np.float64)
        rc = self.lib.oracle_oproj_rows(B, T, d_model, h, g, d_h, k, dt, _ptr(oa), _ptr(wa), _ptr(ia),
                                        ra.shape[0], _ptr(ra), _ptr(out), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_oproj_rows failed ({rc})")
        return out

    def decode_paged(self, q, K_pages, V_pages, block_table, lengths, idx, gate, n_threads=None):
        """Paged GQE decode output O [B, h, d_h] (float64): caches as pages
        [num_pages, page_size, g, d_h], block_table [B, max_blocks], lengths [B]."""
        qa, dt = _as_input(q)
        ka, dk = _as_input(K_pages)
        va, dv = _as_input(V_pages)
        if not (dt == dk == dv):
            raise TypeError("q and the pages must share a dtype")
        num_pages, page_size, g, d_h = ka.shape
        B = int(np.asarray(lengths).shape[0])
        h = qa.shape[-2]
        ta = np.ascontiguousarray(np.asarray(block_table), dtype=np.int32).reshape(B, -1)
        ia = np.ascontiguousarray(idx, dtype=np.int32).reshape(B, g, -1)
        ga = np.ascontiguousarray(gate, dtype=np.float64).reshape(B, g, -1)
        k = ia.shape[-1]
        la = np.ascontiguousarray(np.asarray(lengths), dtype=np.int32).reshape(B)
        out = np.empty((B, h, d_h), np.float64)
        rc = self.lib.oracle_decode_paged(B, page_size, ta.shape[1], num_pages, h, g, d_h, k, dt, _ptr(qa), _ptr(ka),
                                          _ptr(va), _ptr(ta), _ptr(la), _ptr(ia), _ptr(ga), _ptr(out),
                                          _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_decode_paged failed ({rc})")
        return out

    def attn_backward(self, Q, K, V, idx, gate, dO, t_min=0, n_threads=None):
        """Backward of the routed attention for output gradient dO [B, T, h, d_h]:
        returns (dQ [B,T,h,d_h], dK [B,T,g,d_h], dV [B,T,g,d_h], dgate [B,T,g,k]),
        all float64.  With t_min > 0 only query rows t >= t_min contribute: key
        rows s >= t_min of dK/dV and query rows t >= t_min of dQ/dgate are then
        exact (earlier key rows hold a partial sum, earlier query rows 0)."""
        qa, dt = _as_input(Q)
        ka, dk = _as_input(K)
        va, dv = _as_input(V)
        if not (dt == dk == dv):
            raise TypeError("Q, K and V must share a dtype")
        B, T, h, d_h = qa.shape
        g = ka.shape[2]
        ia = np.ascontiguousarray(idx, dtype=np.int32).reshape(B, T, g, -1)
        ga = np.ascontiguousarray(gate, dtype=np.float64).reshape(B, T, g, -1)
        k = ia.shape[-1]
        da = np.ascontiguousarray(np.asarray(dO, dtype=np.float64)).reshape(B, T, h, d_h)
        dQ = np.empty((B, T, h, d_h), np.float64)
        dK = np.empty((B, T, g, d_h), np.float64)
        dV = np.empty((B, T, g, d_h), np.float64)
        dgate = np.empty((B, T, g, k), np.float64)
        rc = self.lib.oracle_attn_backward(B, T, h, g, d_h, k, dt, int(t_min), _ptr(qa), _ptr(ka), _ptr(va), _ptr(ia), _ptr(ga),
                                           _ptr(da), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dgate), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_attn_backward failed ({rc})")
        return dQ, dK, dV, dgate

    def route_backward(self, x, W_r, idx, gate, dgate, n_threads=None):
        """Router backward for gate gradient dgate [..., g, k]: returns
        (dlogits [..., h], dx [..., d_model], dW_r [d_model, h], dbias [h]),
        all float64."""
        xa, dt = _as_input(x)
        wa, dt2 = _as_input(W_r)
        if dt != dt2:
            raise TypeError("x and W_r must share a dtype")
        lead = xa.shape[:-1]
        d_model = xa.shape[-1]
        h = wa.shape[1]
        BT = int(np.prod(lead)) if lead else 1
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        g, k = ia.shape[-2], ia.shape[-1]
        ia = ia.reshape(BT, g, k)
        ga = np.ascontiguousarray(gate, dtype=np.float64).reshape(BT, g, k)
        dga = np.ascontiguousarray(dgate, dtype=np.float64).reshape(BT, g, k)
        dl = np.empty((BT, h), np.float64)
        dx = np.empty((BT, d_model), np.float64)
        dW = np.empty((d_model, h), np.float64)
        db = np.empty((h,), np.float64)
        rc = self.lib.oracle_route_backward(BT, d_model, h, g, k, dt, _ptr(xa), _ptr(wa), _ptr(ia), _ptr(ga),
                                            _ptr(dga), _ptr(dl), _ptr(dx), _ptr(dW), _ptr(db), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_route_backward failed ({rc})")
        return dl.reshape(*lead, h), dx.reshape(*lead, d_model), dW, db

    def aux_loss(self, logits, idx):
        """Load-balancing auxiliary loss for fp32 router logits [..., h] and the
        selection idx [..., g, k]: returns (loss, dlogits [..., h] float64)."""
        la = np.ascontiguousarray(np.asarray(logits, dtype=np.float32))
        h = la.shape[-1]
        lead = la.shape[:-1]
        N = int(np.prod(lead)) if lead else 1
        ia = np.ascontiguousarray(idx, dtype=np.int32)
        g, k = ia.shape[-2], ia.shape[-1]
        loss = ctypes.c_double()
        dl = np.empty((N, h), np.float64)
        rc = self.lib.oracle_aux_loss(N, h, g, k, _ptr(la), _ptr(ia.reshape(N, g, k)), ctypes.byref(loss), _ptr(dl))
        if rc:
            raise ValueError(f"oracle_aux_loss failed ({rc})")
        return loss.value, dl.reshape(*lead, h)

    def attn(self, Q, K, V, idx, gate, n_threads=None):
        """Full GQE output O [B, T, h, d_h] (float64)."""
        B, T, h, d_h = tuple(Q.shape)
        return self.attn_rows(Q, K, V, idx, gate, None, n_threads).reshape(B, T, h, d_h)

    def decode(self, q, K_cache, V_cache, lengths, idx, gate, n_threads=None):
        """GQE decode output O [B, h, d_h] (float64) for q [B, h, d_h] (or
        [B,1,h,d_h]), caches [B, Lmax, g, d_h], lengths [B], idx/gate [B, g, k]."""
        qa, dt = _as_input(q)
        ka, dk = _as_input(K_cache)
        va, dv = _as_input(V_cache)
        if not (dt == dk == dv):
            raise TypeError("q and the caches must share a dtype")
        B, Lmax, g, d_h = ka.shape
        h = qa.shape[-2]
        ia = np.ascontiguousarray(idx, dtype=np.int32).reshape(B, g, -1)
        ga = np.ascontiguousarray(gate, dtype=np.float64).reshape(B, g, -1)
        k = ia.shape[-1]
        la = np.ascontiguousarray(np.asarray(lengths), dtype=np.int32).reshape(B)
        out = np.empty((B, h, d_h), np.float64)
        rc = self.lib.oracle_decode(B, Lmax, h, g, d_h, k, dt, _ptr(qa), _ptr(ka), _ptr(va),
                                    _ptr(la), _ptr(ia), _ptr(ga), _ptr(out), _threads(n_threads))
        if rc:
            raise ValueError(f"oracle_decode failed ({rc})")
        return out


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def route(*a, **kw):
    return default().route(*a, **kw)


def compact(*a, **kw):
    return default().compact(*a, **kw)


def attn_rows(*a, **kw):
    return default().attn_rows(*a, **kw)


def attn(*a, **kw):
    return default().attn(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def shared_rows(*a, **kw):
    return default().shared_rows(*a, **kw)


def group_slots_rows(*a, **kw):
    return default().group_slots_rows(*a, **kw)


def qproj_rows(*a, **kw):
    return default().qproj_rows(*a, **kw)


def oproj_rows(*a, **kw):
    return default().oproj_rows(*a, **kw)


def decode_paged(*a, **kw):
    return default().decode_paged(*a, **kw)


def attn_backward(*a, **kw):
    return default().attn_backward(*a, **kw)


def route_backward(*a, **kw):
    return default().route_backward(*a, **kw)


def aux_loss(*a, **kw):
    return default().aux_loss(*a, **kw)
