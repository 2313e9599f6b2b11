"""The C-ABI library builds, loads and exports every entry point that
include/gqe.h declares; host-side validation rejects bad arguments before any
CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from routed_head_gqa_b200 import build as gqe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqe.h")


@pytest.fixture(scope="module")
def lib():
    path = gqe_build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for required in ("gqe_route", "gqe_attn_prefill", "gqe_attn_decode"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in gqe.h but not exported"


def test_binding_names_match_header():
    import routed_head_gqa_b200 as g

    for name in declared_functions():
        assert callable(getattr(g, name)), f"binding lacks {name}"
    assert sorted(g.EXPORTED) == declared_functions()


def test_status_strings_and_chunks():
    import routed_head_gqa_b200 as g

    assert g.gqe_status_string(g.GQE_OK) == "GQE_OK"
    assert g.gqe_status_string(g.GQE_ERR_DEVICE_TIMEOUT) == "GQE_ERR_DEVICE_TIMEOUT"
    assert g.gqe_status_string(99) == "GQE_UNKNOWN_STATUS"
    assert [g.gqe_chunk_count(t) for t in (0, 1, 32, 33, 4096)] == [0, 1, 1, 2, 128]


def test_workspace_bytes():
    import routed_head_gqa_b200 as g

    s = g.make_shape(8, 4096, 4096, 32, 8, 128, 2, g.GQE_BF16)
    n = g.gqe_workspace_bytes(s, 0)
    assert n >= 256 + 8 * 32 * 128 * 4
    assert g.gqe_workspace_bytes(s, 16384) >= n
    bad = g.make_shape(8, 4096, 4096, 30, 8, 128, 2, g.GQE_BF16)  # h % g != 0
    assert g.gqe_workspace_bytes(bad, 0) == 0


@pytest.mark.parametrize("field,value,code", [
    ("h", 30, 1),       # h % g != 0
    ("k", 5, 1),        # k > h/g
    ("k", 0, 1),
    ("T", 0, 1),
    ("B", 0, 1),        # empty batch: rejected before anything is enqueued
    ("dtype", 7, 1),
])
def test_route_rejects_bad_shapes(field, value, code):
    import routed_head_gqa_b200 as g

    s = g.make_shape(2, 64, 128, 32, 8, 128, 2, g.GQE_BF16)
    setattr(s, field, value)
    fake = 0x10000  # never dereferenced: validation fails first
    rc = g._lib.gqe_route(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, fake, fake, 1 << 20, None)
    assert rc == code


def test_null_and_misaligned_pointers_rejected():
    import routed_head_gqa_b200 as g

    s = g.make_shape(2, 64, 128, 32, 8, 128, 2, g.GQE_BF16)
    fake = 0x10000
    assert g._lib.gqe_route(ctypes.byref(s), None, fake, None, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 1
    assert g._lib.gqe_route(ctypes.byref(s), fake + 2, fake, None, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 1
    # workspace too small / misaligned
    assert g._lib.gqe_route(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, fake, fake, 16, None) == 1
    assert g._lib.gqe_route(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, fake, fake + 16, 1 << 20, None) == 1
    assert g._lib.gqe_attn_prefill(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                   1 << 20, None) == 1
    # decode requires T == 1 and Lmax >= 1
    assert g._lib.gqe_attn_decode(ctypes.byref(s), fake, fake, fake, 128, fake, fake, fake, fake, fake,
                                  1 << 30, None) == 1
    s1 = g.make_shape(2, 1, 128, 32, 8, 128, 2, g.GQE_BF16)
    assert g._lib.gqe_attn_decode(ctypes.byref(s1), fake, fake, fake, 0, fake, fake, fake, fake, fake,
                                  1 << 30, None) == 1


def test_output_construction_validation():
    import routed_head_gqa_b200 as g

    s = g.make_shape(2, 64, 128, 32, 8, 128, 2, g.GQE_BF16)
    fake = 0x10000
    big = 1 << 30
    # shared head: kv_group outside [0, g), null query, too small a workspace
    for kv in (-1, 8):
        assert g._lib.gqe_attn_shared_head(ctypes.byref(s), fake, fake, fake, kv, fake, fake, big, None) == 1
    assert g._lib.gqe_attn_shared_head(ctypes.byref(s), None, fake, fake, 0, fake, fake, big, None) == 1
    assert g._lib.gqe_attn_shared_head(ctypes.byref(s), fake, fake, fake, 0, fake, fake, 256, None) == 1
    # the workspace of gqe_workspace_bytes covers the shared head's identity tables
    assert g.gqe_workspace_bytes(s, 0) >= 256 + 3 * 2 * 64 * 4 + 3 * 4 + 2 * 2 * 4
    # bf16 needs d_h = 128, as the routed prefill
    s64 = g.make_shape(2, 64, 128, 32, 8, 64, 2, g.GQE_BF16)
    assert g._lib.gqe_attn_shared_head(ctypes.byref(s64), fake, fake, fake, 0, fake, fake, big, None) == 2
    # group slots: at least one output, supported d_h
    assert g._lib.gqe_group_slots(ctypes.byref(s), fake, fake, fake, None, None, None) == 1
    assert g._lib.gqe_group_slots(ctypes.byref(s), None, fake, fake, fake, fake, None) == 1
    assert g._lib.gqe_group_slots(ctypes.byref(s), fake, fake, fake, fake + 8, None, None) == 1
    s96 = g.make_shape(2, 64, 128, 32, 8, 96, 2, g.GQE_BF16)
    assert g._lib.gqe_group_slots(ctypes.byref(s96), fake, fake, fake, fake, None, None) == 2


def test_routed_qproj_validation():
    import routed_head_gqa_b200 as g

    fake = 0x10000
    s = g.make_shape(2, 64, 128, 32, 8, 128, 2, g.GQE_BF16)
    call = lambda s, x, W, idx: g._lib.gqe_routed_qproj(ctypes.byref(s), x, W, idx, fake, fake, fake, fake, 1 << 20,
                                                        None)
    assert call(s, None, fake, fake) == 1
    assert call(s, fake, fake + 4, fake) == 1
    assert call(s, fake, fake, None) == 1        # no idx
    assert call(s, fake, fake, fake + 4) == 1    # misaligned idx
    # tensor-core path only: bf16 with d_h = 128
    s32 = g.make_shape(2, 64, 128, 32, 8, 128, 2, g.GQE_F32)
    assert call(s32, fake, fake, fake) == 2
    s64 = g.make_shape(2, 64, 128, 32, 8, 64, 2, g.GQE_BF16)
    assert call(s64, fake, fake, fake) == 2


def test_routed_oproj_validation():
    import routed_head_gqa_b200 as g

    fake = 0x10000
    call = lambda s, O, idx, W, Y, ws=1 << 20: g._lib.gqe_routed_oproj(ctypes.byref(s), O, idx, W, Y, fake, ws,
                                                                       None)
    s = g.make_shape(2, 64, 256, 32, 8, 128, 2, g.GQE_BF16)
    assert call(s, None, fake, fake, fake) == 1          # no O
    assert call(s, fake, None, fake, fake) == 1          # no idx
    assert call(s, fake, fake + 4, fake, fake) == 1      # misaligned idx
    assert call(s, fake, fake, fake + 8, fake) == 1      # misaligned W_Z
    assert call(s, fake, fake, fake, fake, 16) == 1      # workspace below the status word
    assert call(g.make_shape(2, 64, 256, 32, 8, 128, 2, g.GQE_F32), fake, fake, fake, fake) == 2  # fp32
    assert call(g.make_shape(2, 64, 256, 32, 8, 96, 2, g.GQE_BF16), fake, fake, fake, fake) == 2  # d_h 96
    assert call(g.make_shape(2, 64, 256, 128, 8, 128, 2, g.GQE_BF16), fake, fake, fake, fake) == 2  # h > 64
    assert call(g.make_shape(2, 64, 200, 32, 8, 128, 2, g.GQE_BF16), fake, fake, fake, fake) == 2  # d_model % 32


def test_decode_paged_validation():
    import routed_head_gqa_b200 as g

    fake = 0x10000
    s1 = g.make_shape(2, 1, 128, 32, 8, 128, 2, g.GQE_BF16)
    big = 1 << 30
    call = lambda s, npages, ps, bt, nb: g._lib.gqe_attn_decode_paged(
        ctypes.byref(s), fake, fake, fake, npages, ps, bt, nb, fake, fake, fake, fake, fake, big, None)
    assert call(s1, 16, 48, fake, 4) == 1      # page size not a power of two
    assert call(s1, 16, 0, fake, 4) == 1
    assert call(s1, 0, 64, fake, 4) == 1       # empty pool
    assert call(s1, 16, 64, None, 4) == 1      # no block table
    s2 = g.make_shape(2, 2, 128, 32, 8, 128, 2, g.GQE_BF16)
    assert call(s2, 16, 64, fake, 4) == 1      # decode: T must be 1


def test_attn_backward_validation():
    import routed_head_gqa_b200 as g

    fake = 0x10000
    a256 = lambda n: (n + 255) // 256 * 256
    # fp32 inputs (CUDA-core backward): status word + the larger of the attention
    # scratch (gate, D, lse per (b,t,j)) and the router's dW_r partials
    s32 = g.make_shape(2, 64, 128, 8, 2, 128, 2, g.GQE_F32)
    assert g.gqe_backward_workspace_bytes(s32) == 256 + max(3 * 2 * 64 * 8 * 4, 64 * 128 * 8 * 4)
    # bf16 with d_h = 128 (tensor-core backward): the lse plane and the rows'
    # fp32 outputs of the forward recompute, then the packed half-window tiles
    # (2*ceil(T/2W) per (b, group), W = 64 for k = 2): 2 KB tables, Q and dO rows
    s = g.make_shape(2, 64, 128, 8, 2, 128, 2, g.GQE_BF16)
    need = g.gqe_backward_workspace_bytes(s)
    bth, tiles = 2 * 64 * 8, 2 * 2 * 2
    attn = a256(bth * 4) + a256(bth * 128 * 4) + a256(tiles * 2048) + 2 * a256(tiles * 128 * 128 * 2)
    assert need == 256 + max(attn, 64 * 128 * 8 * 4)
    call = lambda s, dQ, ws_bytes: g._lib.gqe_attn_prefill_backward(
        ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, fake, dQ, fake, fake, fake, fake,
        ws_bytes, None)
    assert call(s, None, need) == 1             # no dQ
    assert call(s, fake + 8, need) == 1         # misaligned dQ
    assert call(s, fake, 256 + attn - 1) == 1   # workspace too small for the attention scratch
    train = lambda s, o32, lse: g._lib.gqe_attn_prefill_train(
        ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, None, o32, lse, fake, 1 << 20, None)
    assert train(s, None, fake) == 1            # no O32
    assert train(s, fake, None) == 1            # no lse
    assert train(s32, fake, fake) == 2          # the training forward is the tensor-core path only
    saved = lambda s, lse, ws_bytes: g._lib.gqe_attn_prefill_backward_saved(
        ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, lse, fake, fake, fake, fake,
        fake, ws_bytes, None)
    assert saved(s, None, need) == 1            # no lse
    assert saved(s, fake, 256 + attn - 1) == 1  # workspace too small
    assert saved(s32, fake, 1 << 30) == 2       # fp32: no saved-statistics path
    s96 = g.make_shape(2, 64, 128, 8, 2, 96, 2, g.GQE_BF16)
    assert call(s96, fake, 1 << 30) == 2        # d_h 96 not implemented
    bad = g.make_shape(2, 64, 128, 8, 3, 128, 2, g.GQE_BF16)
    assert call(bad, fake, 1 << 30) == 1        # h % g != 0
    assert g.gqe_backward_workspace_bytes(bad) == 0
    rcall = lambda s, dx, ws_bytes: g._lib.gqe_route_backward(ctypes.byref(s), fake, fake, fake, dx, fake, None,
                                                              fake, ws_bytes, None)
    assert rcall(s, None, need) == 1            # no dx
    assert rcall(s, fake, 255) == 1             # workspace too small
    assert rcall(s, fake + 4, need) == 1        # misaligned dx
    huge = g.make_shape(1 << 13, 1 << 10, 128, 8, 2, 128, 2, g.GQE_BF16)
    assert rcall(huge, fake, 1 << 40) == 2      # more tokens than the dx grid covers


def test_unsupported_cases_report_unsupported():
    import routed_head_gqa_b200 as g

    fake = 0x10000
    # bf16 prefill is implemented for d_h = 128 only
    s = g.make_shape(2, 64, 128, 8, 2, 64, 2, g.GQE_BF16)
    assert g._lib.gqe_attn_prefill(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                   1 << 20, None) == 2
    # decode: d_h 96 not implemented
    s = g.make_shape(2, 1, 128, 8, 2, 96, 2, g.GQE_BF16)
    assert g._lib.gqe_attn_decode(ctypes.byref(s), fake, fake, fake, 64, fake, fake, fake, fake, fake,
                                  1 << 30, None) == 2


def test_kv_cache_ratio_golden():
    """The decode byte accounting reproduces the pages' KV-cache reduction
    (32 query heads over 8 KV groups -> 4x smaller cache than MHA)."""
    from routed_head_gqa_b200 import metrics
    from tests.oracle_pins import read_golden

    h, g_, ratio = read_golden("kv_cache_ratio.txt")[0]
    mha = metrics.kv_cache_bytes(n_kv=h, d_h=128, T=4096)
    gqa = metrics.kv_cache_bytes(n_kv=g_, d_h=128, T=4096)
    assert mha == ratio * gqa
