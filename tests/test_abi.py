"""The C ABI library loads, exports every symbol include/vsa.h declares, and
rejects bad arguments on the host before any CUDA call (runs without a GPU)."""
import ctypes
import os
import re

import pytest

import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import _lib, Shape, MaskParams

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vsa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = _lib.load()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.vsa_version().decode().count(".") == 2


def _call_flatten(shape, x=1 << 12, y=1 << 20):
    L = _lib.load()
    return L.vsa_fractal_flatten(ctypes.c_void_p(x), ctypes.c_void_p(y), shape, None)


@pytest.mark.parametrize("shape,status", [
    (Shape(1, 2, 4, 16, 16, 96), 2),     # d not 64/128
    (Shape(1, 2, 4, 16, 16, 64, P=4), 2),  # P*P != 64
    (Shape(1, 2, 4, 12, 16, 64), 2),     # H not a multiple of P
    (Shape(-1, 2, 4, 16, 16, 64), 1),    # negative size
])
def test_shape_validation(shape, status):
    assert _call_flatten(shape.c()) == status
    assert len(_lib.load().vsa_last_error()) > 0


def test_null_and_misaligned_pointers_rejected():
    s = Shape(1, 2, 4, 16, 16, 64).c()
    assert _call_flatten(s, x=0) == 1
    assert _call_flatten(s, x=(1 << 12) + 8) == 2
    assert _call_flatten(s, x=1 << 12, y=(1 << 12) + 64) == 1   # overlapping buffers


def test_mask_parameter_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64)
    P = ctypes.c_void_p
    def call(params, cap=2 * 16 * 16, ws=1 << 30):
        return L.vsa_block_mask(P(1 << 12), P(1 << 16), s.c(), params.c(), P(1 << 20), P(1 << 24),
                                cap, None, P(1 << 28), ws, None)
    assert call(MaskParams(1.0)) == 1
    assert call(MaskParams(-0.1)) == 1
    assert call(MaskParams(0.2, True, (1, -1, 1))) == 1
    assert call(MaskParams(0.2), cap=2 * 16 * 16 - 1) == 3          # CSR capacity
    assert call(MaskParams(0.2), ws=16) == 3                        # workspace
    assert _lib.load().vsa_block_mask_workspace_size(Shape(1, 1, 1, 8, 8, 96).c()) == 0


def test_attention_workspace_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64)
    P = ctypes.c_void_p
    st = L.vsa_sparse_attn_fwd(P(1 << 12), P(1 << 16), P(1 << 20), P(1 << 24), P(1 << 26), s.c(),
                               0.0, P(1 << 28), P(1 << 29), P(1 << 30), 8, None)
    assert st == 3
    assert L.vsa_sparse_attn_workspace_size(s.c()) > 0


def test_flatten_pool_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64).c()          # 256 KiB per bf16 tensor
    P = ctypes.c_void_p
    MB = 1 << 20
    def call(q=1 * MB, k=2 * MB, qf=3 * MB, kf=4 * MB, qp=5 * MB, kp=6 * MB):
        return L.vsa_flatten_pool_qk(P(q), P(k), P(qf), P(kf), P(qp), P(kp), s, None)
    assert call(q=0) == 1
    assert call(kp=0) == 1
    assert call(qf=3 * MB + 8) == 2                 # misaligned
    assert call(qf=1 * MB + 4096) == 1              # output inside an input
    assert call(kf=3 * MB + 65536) == 1             # two outputs overlap
    assert call(qp=4 * MB + 128 * 1024) == 1        # pooled output inside kf
    assert len(L.vsa_last_error()) > 0


def test_static_ratio_and_sta_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64)              # Nb = 16 per head, 32 rows
    P = ctypes.c_void_p
    def topk(k, cap=2 * 16 * 16, ws=1 << 30, params=MaskParams(0.0, True)):
        return L.vsa_block_mask_topk(P(1 << 12), P(1 << 16), s.c(), k, params.c(), P(1 << 20),
                                     P(1 << 24), cap, None, P(1 << 28), ws, None)
    assert topk(0) == 1                                     # k < 1
    assert topk(-3) == 1
    assert topk(4, params=MaskParams(0.0, True, (1, -1, 0))) == 1
    assert topk(4, cap=2 * 16 * 16 - 1) == 3                # CSR capacity
    assert topk(4, ws=16) == 3                              # workspace
    def sta(r=(1, 1, 1), cap=1 << 20):
        return L.vsa_sta_mask(s.c(), r[0], r[1], r[2], P(1 << 20), P(1 << 24), cap, None, None)
    assert sta((-1, 0, 0)) == 1
    need = vsa.sta_mask_nnz(s, (1, 1, 1))
    # 2 heads x (sum of clipped widths: 4 frames -> 2+3+3+2, 2 patch rows -> 2+2, 2 cols -> 2+2)
    assert need == 2 * 10 * 4 * 4
    assert sta(cap=need - 1) == 3
    assert len(L.vsa_last_error()) > 0


def test_query_subset_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64)              # 32 query blocks
    P = ctypes.c_void_p
    def call(qb, n):
        return L.vsa_sparse_attn_fwd_rows(P(1 << 12), P(1 << 16), P(1 << 20), P(1 << 24),
                                          P(1 << 26), s.c(), 0.0, qb, n, P(1 << 28), P(1 << 29),
                                          P(1 << 30), 1 << 20, None)
    assert call(P(1 << 12), -1) == 1
    assert call(None, 4) == 1                   # null list
    assert call(P((1 << 12) + 2), 4) == 1       # misaligned list
    assert call(P(1 << 12), 33) == 1            # more entries than query blocks
    assert call(None, 0) == 0                   # nothing to do


def test_raster_pool_and_attention_validation():
    L = _lib.load()
    s = Shape(1, 2, 4, 16, 16, 64)              # 256 KiB per bf16 tensor, 16 KiB pooled
    P = ctypes.c_void_p
    MB = 1 << 20
    def pool(q=1 * MB, k=2 * MB, qp=3 * MB, kp=4 * MB):
        return L.vsa_pool_qk_raster(P(q), P(k), P(qp), P(kp), s.c(), None)
    assert pool(q=0) == 1
    assert pool(kp=0) == 1
    assert pool(qp=3 * MB + 8) == 2                 # misaligned
    assert pool(qp=1 * MB + 4096) == 1              # output inside an input
    assert pool(kp=3 * MB + 4096) == 1              # the two outputs overlap
    def attn(ws_bytes=1 << 20, q=1 << 12, lse=1 << 29):
        return L.vsa_sparse_attn_fwd_raster(P(q), P(1 << 16), P(1 << 20), P(1 << 24), P(1 << 26),
                                            s.c(), 0.0, P(1 << 28), P(lse), P(1 << 30), ws_bytes,
                                            None)
    assert attn(q=0) == 1
    assert attn(q=(1 << 12) + 8) == 2
    assert attn(lse=(1 << 29) + 2) == 2
    assert attn(ws_bytes=8) == 3                    # workspace too small
    assert len(L.vsa_last_error()) > 0
    # flattened inputs, raster outputs: the same checks before any launch
    def to_raster(ws_bytes=1 << 20, q=1 << 12, lse=1 << 29):
        return L.vsa_sparse_attn_fwd_to_raster(P(q), P(1 << 16), P(1 << 20), P(1 << 24),
                                               P(1 << 26), s.c(), 0.0, P(1 << 28), P(lse),
                                               P(1 << 30), ws_bytes, None)
    assert to_raster(q=0) == 1
    assert to_raster(q=(1 << 12) + 8) == 2
    assert to_raster(lse=(1 << 29) + 2) == 2
    assert to_raster(ws_bytes=8) == 3


def test_layer_layout_is_checked_before_allocating():
    with pytest.raises(ValueError, match="layout"):
        vsa.Layer(Shape(1, 2, 4, 16, 16, 64), MaskParams(0.2), "cpu", layout="fractal")


def test_raster_entry_points_accept_an_empty_shape():
    L = _lib.load()
    s = Shape(1, 2, 0, 16, 16, 64).c()            # T = 0: nothing to do, nothing touched
    assert L.vsa_pool_qk_raster(None, None, None, None, s, None) == 0
    assert L.vsa_sparse_attn_fwd_raster(None, None, None, None, None, s, 0.0, None, None, None,
                                        0, None) == 0
    assert L.vsa_sparse_attn_fwd_to_raster(None, None, None, None, None, s, 0.0, None, None,
                                           None, 0, None) == 0


def test_wait_probe_limit_validated_on_the_host():
    L = _lib.load()
    assert L.vsa_wait_probe(0, None) == 1
    assert L.vsa_wait_probe((1 << 32) + 1, None) == 1
    assert b"wait_cycles" in L.vsa_last_error()
