"""Algorithmic work counts for the roofline of the GQE kernels.

Prefill (tensor cores): active-head FLOPs.  Each routed (b, t, j) takes a
causal dot-product row over keys 0..t: QK^T and P.V each cost 2*d_h FLOPs per
key, so the row costs 4*d_h*(t+1).  Unselected heads and the masked upper
triangle are not counted.

Decode (HBM): the KV-cache bytes read.  Per sequence and layer the cache holds
2 * n_kv * d_h * T elements (ml-canon "56 GQA / MQA", KV-cache formula); GQE
keeps the KV path dense, so decode reads all of it once.
"""
from __future__ import annotations

import torch


def kv_cache_bytes(n_kv: int, d_h: int, T: int, layers: int = 1, elem_bytes: int = 2) -> int:
    """Bytes of a KV cache: 2 (K and V) * layers * n_kv * d_h * T elements."""
    return 2 * layers * n_kv * d_h * T * elem_bytes


def prefill_active_flops(B: int, T: int, g: int, k: int, d_h: int) -> int:
    """Active-head FLOPs of a routed prefill.  Every token selects exactly k
    heads per group, so the count depends only on the shape:
    4*d_h * B*g*k * sum_{t<T} (t+1)."""
    return 4 * d_h * B * g * k * (T * (T + 1) // 2)


def prefill_active_flops_from_routing(idx: torch.Tensor, d_h: int) -> int:
    """Same count taken from a realised routing idx [B, T, g, k] (a check of the
    closed form above)."""
    B, T, g, k = idx.shape
    t = torch.arange(T, device=idx.device, dtype=torch.int64) + 1
    valid = (idx >= 0).to(torch.int64).sum(dim=(2, 3))  # [B, T]
    return int(4 * d_h * (valid * t).sum().item())


def decode_kv_bytes(lengths: torch.Tensor, g: int, d_h: int, elem_bytes: int = 2) -> int:
    """Bytes of KV cache a decode step reads: sum_b 2*g*d_h*L_b*elem_bytes."""
    return int(lengths.to(torch.int64).sum().item()) * 2 * g * d_h * elem_bytes


def route_bytes(B: int, T: int, d_model: int, h: int, g: int, k: int, elem_bytes: int = 2) -> int:
    """Bytes the router must move: x and W_r read, idx and gate written."""
    return (B * T * d_model + d_model * h) * elem_bytes + B * T * g * k * 8


def prefill_io_bytes(B: int, T: int, h: int, g: int, k: int, d_h: int, elem_bytes: int = 2) -> int:
    """Compulsory prefill traffic: routed Q rows, K and V once, O written in full."""
    return (B * T * g * k * d_h + 2 * B * T * g * d_h + B * T * h * d_h) * elem_bytes
