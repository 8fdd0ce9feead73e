"""ctypes binding of libvsa.so (argument marshalling only).

Every function here forwards to the C ABI declared in include/vsa.h; no step
of the computation runs in Python.  Loading fails loudly when the library is
missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvsa.so")

VSA_OK = 0
STATUS_NAMES = {0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_UNSUPPORTED",
                3: "VSA_ERR_CAPACITY", 4: "VSA_ERR_CUDA", 5: "VSA_ERR_DEVICE_TIMEOUT"}

# Every symbol include/vsa.h declares.
EXPORTS = ("vsa_fractal_flatten", "vsa_fractal_unflatten", "vsa_pool_qk",
           "vsa_flatten_pool_qk", "vsa_pool_qk_raster",
           "vsa_block_mask_workspace_size", "vsa_block_mask", "vsa_block_mask_topk",
           "vsa_sta_mask",
           "vsa_sparse_attn_workspace_size", "vsa_sparse_attn_fwd",
           "vsa_sparse_attn_fwd_noalloc", "vsa_sparse_attn_fwd_rows",
           "vsa_sparse_attn_fwd_raster", "vsa_sparse_attn_fwd_to_raster",
           "vsa_cluster_attn_workspace_size", "vsa_cluster_attn_fwd",
           "vsa_last_error", "vsa_device_status", "vsa_wait_probe", "vsa_version")


class vsa_cluster_params(ctypes.Structure):
    _fields_ = [("Cq", ctypes.c_int32), ("Ck", ctypes.c_int32), ("iters", ctypes.c_int32),
                ("p", ctypes.c_float)]


class vsa_cluster_state(ctypes.Structure):
    _fields_ = [("q_labels", ctypes.c_void_p), ("k_labels", ctypes.c_void_p),
                ("q_counts", ctypes.c_void_p), ("k_counts", ctypes.c_void_p),
                ("q_centroids", ctypes.c_void_p), ("k_centroids", ctypes.c_void_p),
                ("keep", ctypes.c_void_p)]


class vsa_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("d", ctypes.c_int32),
                ("P", ctypes.c_int32)]


class vsa_mask_params(ctypes.Structure):
    _fields_ = [("thr", ctypes.c_float), ("use_sta", ctypes.c_int32),
                ("sta_t", ctypes.c_int32), ("sta_h", ctypes.c_int32), ("sta_w", ctypes.c_int32)]


class VsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load():
    """Load libvsa.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    from . import build as _build
    if not os.path.exists(LIB_PATH) or _build._stale():
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libvsa.so not found at {LIB_PATH}; run "
                          "`python -m content_adaptive_block_fractal_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, S, I64, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_float
    st = ctypes.c_int
    for name, args in {
        "vsa_fractal_flatten": [P, P, vsa_shape, P],
        "vsa_fractal_unflatten": [P, P, vsa_shape, P],
        "vsa_pool_qk": [P, P, P, P, vsa_shape, P],
        "vsa_flatten_pool_qk": [P, P, P, P, P, P, vsa_shape, P],
        "vsa_pool_qk_raster": [P, P, P, P, vsa_shape, P],
        "vsa_block_mask": [P, P, vsa_shape, vsa_mask_params, P, P, I64, P, P, S, P],
        "vsa_block_mask_topk": [P, P, vsa_shape, ctypes.c_int32, vsa_mask_params, P, P, I64, P,
                                P, S, P],
        "vsa_sta_mask": [vsa_shape, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, I64,
                         P, P],
        "vsa_sparse_attn_fwd": [P, P, P, P, P, vsa_shape, F, P, P, P, S, P],
        "vsa_sparse_attn_fwd_raster": [P, P, P, P, P, vsa_shape, F, P, P, P, S, P],
        "vsa_sparse_attn_fwd_to_raster": [P, P, P, P, P, vsa_shape, F, P, P, P, S, P],
        "vsa_sparse_attn_fwd_noalloc": [P, P, P, P, P, vsa_shape, F, P, P, P],
        "vsa_sparse_attn_fwd_rows": [P, P, P, P, P, vsa_shape, F, P, I64, P, P, P, S, P],
        "vsa_device_status": [P],
        "vsa_wait_probe": [I64, P],
        "vsa_cluster_attn_fwd": [P, P, P, vsa_shape, vsa_cluster_params, F, P, P, P, P,
                                 ctypes.POINTER(vsa_cluster_state), P, S, P],
    }.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = st
    L.vsa_block_mask_workspace_size.argtypes = [vsa_shape]
    L.vsa_block_mask_workspace_size.restype = S
    L.vsa_sparse_attn_workspace_size.argtypes = [vsa_shape]
    L.vsa_sparse_attn_workspace_size.restype = S
    L.vsa_cluster_attn_workspace_size.argtypes = [vsa_shape, vsa_cluster_params]
    L.vsa_cluster_attn_workspace_size.restype = S
    L.vsa_last_error.restype = ctypes.c_char_p
    L.vsa_version.restype = ctypes.c_char_p
    _lib = L
    return L


def check(status: int) -> None:
    if status != VSA_OK:
        raise VsaError(status, load().vsa_last_error().decode())
