"""Python binding of libgqe (include/gqe.h): the GQE attention forward pass on B200.

Argument marshalling only.  Every step of the routed path (router, top-k,
compaction, routed prefill, decode) runs in the library's CUDA kernels; PyTorch
supplies device memory and the current CUDA stream.  The functions keep the C
names and raise ``GQEError`` on a non-OK status.  The first call loads
``libgqe.so`` and raises ImportError if it has not been built
(``python -m routed_head_gqa_b200.build``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqe.so")

GQE_OK = 0
GQE_ERR_INVALID_ARGUMENT = 1
GQE_ERR_UNSUPPORTED = 2
GQE_ERR_CUDA = 3
GQE_ERR_DEVICE_TIMEOUT = 4
GQE_ERR_SCRATCH_LIMIT = 5
GQE_F32 = 0
GQE_BF16 = 1

EXPORTED = ["gqe_chunk_count", "gqe_workspace_bytes", "gqe_workspace_init", "gqe_route", "gqe_route_static",
            "gqe_route_static_status",
            "gqe_attn_prefill", "gqe_attn_decode", "gqe_attn_decode_paged", "gqe_attn_shared_head",
            "gqe_group_slots", "gqe_routed_qproj", "gqe_routed_oproj", "gqe_backward_workspace_bytes", "gqe_attn_prefill_backward",
            "gqe_route_backward", "gqe_route_train", "gqe_aux_loss_workspace_bytes", "gqe_aux_loss",
            "gqe_attn_prefill_train", "gqe_attn_prefill_backward_saved",
            "gqe_get_device_status", "gqe_status_string"]


class GqeShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("d_model", ctypes.c_int), ("h", ctypes.c_int),
                ("g", ctypes.c_int), ("d_h", ctypes.c_int), ("k", ctypes.c_int), ("dtype", ctypes.c_int)]


class GQEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {gqe_status_string(status)} ({status})")


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_lib_handle = None


def _load():
    """Load libgqe.so on first use; fail loudly when it has not been built."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m routed_head_gqa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    S = ctypes.POINTER(GqeShape)
    lib.gqe_chunk_count.argtypes = [_I]
    lib.gqe_chunk_count.restype = _I
    lib.gqe_workspace_bytes.argtypes = [S, _I]
    lib.gqe_workspace_bytes.restype = _SZ
    lib.gqe_workspace_init.argtypes = [_P, _SZ, _P]
    lib.gqe_route.argtypes = [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_route_static.argtypes = [S, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.gqe_route_static_status.argtypes = [_P]
    lib.gqe_attn_prefill.argtypes = [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_attn_decode.argtypes = [S, _P, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_attn_shared_head.argtypes = [S, _P, _P, _P, _I, _P, _P, _SZ, _P]
    lib.gqe_group_slots.argtypes = [S, _P, _P, _P, _P, _P, _P]
    lib.gqe_routed_qproj.argtypes = [S, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_routed_oproj.argtypes = [S, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_attn_decode_paged.argtypes = [S, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_backward_workspace_bytes.argtypes = [S]
    lib.gqe_backward_workspace_bytes.restype = _SZ
    lib.gqe_attn_prefill_backward.argtypes = [S] + [_P] * 14 + [_SZ, _P]
    lib.gqe_route_backward.argtypes = [S] + [_P] * 7 + [_SZ, _P]
    lib.gqe_route_train.argtypes = [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_aux_loss_workspace_bytes.argtypes = [S]
    lib.gqe_aux_loss_workspace_bytes.restype = _SZ
    lib.gqe_aux_loss.argtypes = [S, _P, _P, _P, _P, _P, _SZ, _P]
    lib.gqe_attn_prefill_train.argtypes = [S] + [_P] * 12 + [_SZ, _P]
    lib.gqe_attn_prefill_backward_saved.argtypes = [S] + [_P] * 16 + [_SZ, _P]
    lib.gqe_get_device_status.argtypes = [_P, _P]
    lib.gqe_status_string.argtypes = [_I]
    lib.gqe_status_string.restype = ctypes.c_char_p
    for f in ("gqe_workspace_init", "gqe_route", "gqe_route_static", "gqe_route_static_status",
              "gqe_attn_prefill", "gqe_attn_decode",
              "gqe_attn_shared_head", "gqe_group_slots", "gqe_routed_qproj", "gqe_routed_oproj",
              "gqe_attn_decode_paged",
              "gqe_attn_prefill_backward", "gqe_route_backward", "gqe_get_device_status", "gqe_route_train",
              "gqe_aux_loss", "gqe_attn_prefill_train", "gqe_attn_prefill_backward_saved"):
        getattr(lib, f).restype = _I
    _lib_handle = lib
    return lib


class _LazyLib:
    def __getattr__(self, name):
        return getattr(_load(), name)


_lib = _LazyLib()


def make_shape(B, T, d_model, h, g, d_h, k, dtype) -> GqeShape:
    """dtype: GQE_F32 / GQE_BF16 or a torch dtype."""
    if isinstance(dtype, torch.dtype):
        dtype = GQE_BF16 if dtype == torch.bfloat16 else GQE_F32
    return GqeShape(int(B), int(T), int(d_model), int(h), int(g), int(d_h), int(k), int(dtype))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t):
    return t.numel() * t.element_size()


def _check(fn, status):
    if status != GQE_OK:
        raise GQEError(fn, status)


def gqe_status_string(status: int) -> str:
    return _lib.gqe_status_string(int(status)).decode()


def gqe_chunk_count(T: int) -> int:
    return _lib.gqe_chunk_count(int(T))


def gqe_workspace_bytes(shape: GqeShape, Lmax: int = 0) -> int:
    return _lib.gqe_workspace_bytes(ctypes.byref(shape), int(Lmax))


def gqe_workspace_init(workspace, stream=None) -> None:
    _check("gqe_workspace_init", _lib.gqe_workspace_init(_ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_route(shape, x, W_r, bias, idx, gate, head_offsets, head_pos, head_chunk_offsets, workspace,
              stream=None) -> None:
    _check("gqe_route", _lib.gqe_route(ctypes.byref(shape), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(idx),
                                       _ptr(gate), _ptr(head_offsets), _ptr(head_pos),
                                       _ptr(head_chunk_offsets), _ptr(workspace), _nbytes(workspace),
                                       _stream(stream)))


def gqe_route_static(shape, x, W_r, bias, idx, gate, head_offsets, head_pos, head_chunk_offsets,
                     stream=None) -> None:
    """gqe_route with the library's own scratch: no workspace, no allocation.
    For callers that cannot allocate device memory; see include/gqe.h for the
    size limit and the rule that overlapping calls race on the shared scratch."""
    _check("gqe_route_static", _lib.gqe_route_static(ctypes.byref(shape), _ptr(x), _ptr(W_r), _ptr(bias),
                                                     _ptr(idx), _ptr(gate), _ptr(head_offsets), _ptr(head_pos),
                                                     _ptr(head_chunk_offsets), _stream(stream)))


def gqe_route_static_status(stream=None) -> int:
    """Device status of gqe_route_static on the current device (synchronises
    the stream; returns the first recorded error code and clears it)."""
    return _lib.gqe_route_static_status(_stream(stream))


def gqe_attn_prefill(shape, Q, K, V, idx, gate, head_offsets, head_pos, head_chunk_offsets, O, workspace,
                     stream=None) -> None:
    _check("gqe_attn_prefill", _lib.gqe_attn_prefill(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                                     _ptr(gate), _ptr(head_offsets), _ptr(head_pos),
                                                     _ptr(head_chunk_offsets), _ptr(O), _ptr(workspace),
                                                     _nbytes(workspace), _stream(stream)))


def gqe_backward_workspace_bytes(shape) -> int:
    return int(_lib.gqe_backward_workspace_bytes(ctypes.byref(shape)))


def gqe_attn_prefill_backward(shape, Q, K, V, idx, gate, head_offsets, head_pos, head_chunk_offsets, dO, dQ, dK, dV,
                              dlogits, workspace, stream=None) -> None:
    _check("gqe_attn_prefill_backward",
           _lib.gqe_attn_prefill_backward(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(gate),
                                          _ptr(head_offsets), _ptr(head_pos), _ptr(head_chunk_offsets),
                                          _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dlogits), _ptr(workspace),
                                          _nbytes(workspace), _stream(stream)))


def gqe_route_backward(shape, x, W_r, dlogits, dx, dW_r, dbias, workspace, stream=None) -> None:
    _check("gqe_route_backward",
           _lib.gqe_route_backward(ctypes.byref(shape), _ptr(x), _ptr(W_r), _ptr(dlogits), _ptr(dx), _ptr(dW_r),
                                   _ptr(dbias), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_attn_decode(shape, q, K_cache, V_cache, Lmax, lengths, idx, gate, O, workspace, stream=None) -> None:
    _check("gqe_attn_decode", _lib.gqe_attn_decode(ctypes.byref(shape), _ptr(q), _ptr(K_cache), _ptr(V_cache),
                                                   int(Lmax), _ptr(lengths), _ptr(idx), _ptr(gate), _ptr(O),
                                                   _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_attn_shared_head(shape, Qs, K, V, kv_group, Os, workspace, stream=None) -> None:
    _check("gqe_attn_shared_head", _lib.gqe_attn_shared_head(ctypes.byref(shape), _ptr(Qs), _ptr(K), _ptr(V),
                                                             int(kv_group), _ptr(Os), _ptr(workspace),
                                                             _nbytes(workspace), _stream(stream)))


def gqe_attn_decode_paged(shape, q, K_pages, V_pages, page_size, block_table, lengths, idx, gate, O, workspace,
                          stream=None) -> None:
    num_pages = int(K_pages.shape[0])
    max_blocks = int(block_table.shape[-1])
    _check("gqe_attn_decode_paged", _lib.gqe_attn_decode_paged(
        ctypes.byref(shape), _ptr(q), _ptr(K_pages), _ptr(V_pages), num_pages, int(page_size), _ptr(block_table),
        max_blocks, _ptr(lengths), _ptr(idx), _ptr(gate), _ptr(O), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))


def gqe_routed_qproj(shape, x, W_Q, idx, head_offsets, head_pos, Q, workspace, stream=None) -> None:
    _check("gqe_routed_qproj", _lib.gqe_routed_qproj(ctypes.byref(shape), _ptr(x), _ptr(W_Q), _ptr(idx),
                                                     _ptr(head_offsets), _ptr(head_pos), _ptr(Q), _ptr(workspace),
                                                     _nbytes(workspace), _stream(stream)))


def gqe_routed_oproj(shape, O, idx, W_Z, Y, workspace, stream=None) -> None:
    _check("gqe_routed_oproj", _lib.gqe_routed_oproj(ctypes.byref(shape), _ptr(O), _ptr(idx), _ptr(W_Z), _ptr(Y),
                                                     _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_group_slots(shape, O, idx, gate, O_cat, O_wsum, stream=None) -> None:
    _check("gqe_group_slots", _lib.gqe_group_slots(ctypes.byref(shape), _ptr(O), _ptr(idx), _ptr(gate),
                                                   _ptr(O_cat), _ptr(O_wsum), _stream(stream)))


def gqe_route_train(shape, x, W_r, bias, idx, gate, head_offsets, head_pos, head_chunk_offsets, logits, workspace,
                    stream=None) -> None:
    _check("gqe_route_train", _lib.gqe_route_train(ctypes.byref(shape), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(idx),
                                                   _ptr(gate), _ptr(head_offsets), _ptr(head_pos),
                                                   _ptr(head_chunk_offsets), _ptr(logits), _ptr(workspace),
                                                   _nbytes(workspace), _stream(stream)))


def gqe_attn_prefill_train(shape, Q, K, V, idx, gate, head_offsets, head_pos, head_chunk_offsets, O, O32, lse,
                           workspace, stream=None) -> None:
    _check("gqe_attn_prefill_train",
           _lib.gqe_attn_prefill_train(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(gate),
                                       _ptr(head_offsets), _ptr(head_pos), _ptr(head_chunk_offsets), _ptr(O),
                                       _ptr(O32), _ptr(lse), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_attn_prefill_backward_saved(shape, Q, K, V, idx, gate, head_offsets, head_pos, head_chunk_offsets, dO, O32,
                                    lse, dQ, dK, dV, dlogits, workspace, stream=None) -> None:
    _check("gqe_attn_prefill_backward_saved",
           _lib.gqe_attn_prefill_backward_saved(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(gate),
                                                _ptr(head_offsets), _ptr(head_pos), _ptr(head_chunk_offsets), _ptr(dO),
                                                _ptr(O32), _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dlogits),
                                                _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_aux_loss_workspace_bytes(shape) -> int:
    return int(_lib.gqe_aux_loss_workspace_bytes(ctypes.byref(shape)))


def gqe_aux_loss(shape, logits, idx, loss, dlogits, workspace, stream=None) -> None:
    _check("gqe_aux_loss", _lib.gqe_aux_loss(ctypes.byref(shape), _ptr(logits), _ptr(idx), _ptr(loss),
                                             _ptr(dlogits), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def gqe_get_device_status(workspace, stream=None) -> int:
    return _lib.gqe_get_device_status(_ptr(workspace), _stream(stream))


# ---------------------------------------------------------------------------
# Buffer helpers: device memory for the calls above, allocated through torch.
# ---------------------------------------------------------------------------
class Buffers:
    """Routing outputs, O and the workspace for one shape on one device."""

    def __init__(self, shape: GqeShape, device="cuda", Lmax: int = 0):
        B, T, h, g, k, d_h = shape.B, shape.T, shape.h, shape.g, shape.k, shape.d_h
        dt = torch.bfloat16 if shape.dtype == GQE_BF16 else torch.float32
        self.shape = shape
        self.idx = torch.empty((B, T, g, k), dtype=torch.int32, device=device)
        self.gate = torch.empty((B, T, g, k), dtype=torch.float32, device=device)
        self.head_offsets = torch.empty(B * h + 1, dtype=torch.int32, device=device)
        self.head_pos = torch.empty(B * T * g * k, dtype=torch.int32, device=device)
        self.head_chunk_offsets = torch.empty(B * h * gqe_chunk_count(T), dtype=torch.int32, device=device)
        self.O = torch.empty((B, T, h, d_h), dtype=dt, device=device)
        nbytes = gqe_workspace_bytes(shape, Lmax)
        if nbytes == 0:
            raise GQEError("gqe_workspace_bytes", GQE_ERR_INVALID_ARGUMENT)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        gqe_workspace_init(self.workspace)

    def route(self, x, W_r, bias=None, stream=None):
        gqe_route(self.shape, x, W_r, bias, self.idx, self.gate, self.head_offsets, self.head_pos,
                  self.head_chunk_offsets, self.workspace, stream)

    def prefill(self, Q, K, V, stream=None):
        gqe_attn_prefill(self.shape, Q, K, V, self.idx, self.gate, self.head_offsets, self.head_pos,
                         self.head_chunk_offsets, self.O, self.workspace, stream)

    def decode(self, q, K_cache, V_cache, lengths, stream=None):
        gqe_attn_decode(self.shape, q, K_cache, V_cache, K_cache.shape[1], lengths, self.idx, self.gate, self.O,
                        self.workspace, stream)

    def prefill_train(self, Q, K, V, stream=None):
        """The training forward: O as `prefill`, plus each routed row's fp32
        output and log2-sum-exp, kept here for `backward(..., saved=True)`."""
        sh = self.shape
        if getattr(self, "_saved", None) is None:
            f32 = dict(dtype=torch.float32, device=self.idx.device)
            self._saved = (torch.empty((sh.B, sh.T, sh.h, sh.d_h), **f32), torch.empty((sh.B, sh.T, sh.h), **f32))
        O32, lse = self._saved
        gqe_attn_prefill_train(sh, Q, K, V, self.idx, self.gate, self.head_offsets, self.head_pos,
                               self.head_chunk_offsets, self.O, O32, lse, self.workspace, stream)

    def backward(self, Q, K, V, dO, stream=None, saved=False):
        """Gradients of the routed attention for output gradient dO (the routing
        of the last `route`): returns (dQ, dK, dV, dlogits), float32 tensors
        owned by this object and overwritten by the next call.  saved=True
        reads the statistics of the last `prefill_train` instead of
        recomputing the forward."""
        sh = self.shape
        if getattr(self, "_bwd", None) is None:
            dev = self.idx.device
            f32 = dict(dtype=torch.float32, device=dev)
            nbytes = gqe_backward_workspace_bytes(sh)
            self._bwd = (torch.empty((sh.B, sh.T, sh.h, sh.d_h), **f32), torch.empty((sh.B, sh.T, sh.g, sh.d_h), **f32),
                         torch.empty((sh.B, sh.T, sh.g, sh.d_h), **f32), torch.empty((sh.B, sh.T, sh.h), **f32),
                         torch.zeros(nbytes, dtype=torch.uint8, device=dev))
        dQ, dK, dV, dl, ws = self._bwd
        if saved:
            if getattr(self, "_saved", None) is None:
                raise RuntimeError("backward(saved=True) follows prefill_train")
            gqe_attn_prefill_backward_saved(sh, Q, K, V, self.idx, self.gate, self.head_offsets, self.head_pos,
                                            self.head_chunk_offsets, dO, self._saved[0], self._saved[1], dQ, dK, dV,
                                            dl, ws, stream)
        else:
            gqe_attn_prefill_backward(sh, Q, K, V, self.idx, self.gate, self.head_offsets, self.head_pos,
                                      self.head_chunk_offsets, dO, dQ, dK, dV, dl, ws, stream)
        return dQ, dK, dV, dl

    def route_backward(self, x, W_r, dlogits, stream=None):
        """Router gradients (dx, dW_r, dbias) from the logit gradients, float32
        tensors owned by this object (uses the backward workspace)."""
        sh = self.shape
        if getattr(self, "_rbwd", None) is None:
            dev = self.idx.device
            f32 = dict(dtype=torch.float32, device=dev)
            self._rbwd = (torch.empty((sh.B, sh.T, sh.d_model), **f32), torch.empty((sh.d_model, sh.h), **f32),
                          torch.empty((sh.h,), **f32))
        if getattr(self, "_bwd", None) is None:
            raise RuntimeError("route_backward follows backward (it reuses its workspace)")
        dx, dW, db = self._rbwd
        gqe_route_backward(sh, x, W_r, dlogits, dx, dW, db, self._bwd[4], stream)
        return dx, dW, db

    def backward_status(self, stream=None) -> int:
        return gqe_get_device_status(self._bwd[4], stream)

    def status(self, stream=None) -> int:
        return gqe_get_device_status(self.workspace, stream)
