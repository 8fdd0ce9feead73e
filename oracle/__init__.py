"""CPU oracle for content-adaptive block-sparse video attention (fp64).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package.  It
shares no code with the CUDA path; the only thing both sides share is the
seeded input generator, which holds none of the method's arithmetic.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one OpenMP loop over
independent rows); this module only compiles it with gcc and marshals numpy
arrays.  Every function names the page passage it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.oracle_num_threads.restype = _I
        L.oracle_fractal_order.argtypes = [_I, _I, _I, _I, _P]
        L.oracle_flatten.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _I]
        L.oracle_unflatten.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _I]
        L.oracle_unflatten_f64.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _I]
        L.oracle_pool.argtypes = [_P, _P, _I64, _I64, _I, _I]
        L.oracle_reduced_attention.argtypes = [_P, _P, _I64, _I, _I, _P, _I64, _P]
        L.oracle_select_row.argtypes = [_P, _I, _D, _P, _P]
        L.oracle_sta_keep.argtypes = [_I64, _I64, _I, _I, _I, _I, _I]
        L.oracle_sta_keep.restype = _I
        L.oracle_block_mask.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _D, _I, _I,
                                        _I, _I, _P, _I64, _P, _P]
        L.oracle_select_topk_row.argtypes = [_P, _I, _I, _P, _P]
        L.oracle_block_mask_topk.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _I, _I, _I,
                                             _I, _I, _P, _I64, _P, _P]
        L.oracle_sta_mask.argtypes = [_I, _I, _I, _I, _I, _I, _P]
        L.oracle_kmeans_assign.argtypes = [_P, _P, _I64, _I, _I, _P, _P]
        L.oracle_kmeans_update.argtypes = [_P, _P, _I64, _I, _I, _P, _P]
        L.oracle_cluster_order.argtypes = [_P, _I64, _I, _P, _P]
        L.oracle_centroid_topp.argtypes = [_P, _P, _P, _I, _I, _I, _D, _P, _P]
        L.oracle_cluster_attention.argtypes = [_P, _P, _P, _I64, _I, _P, _P, _P, _I, _D, _P,
                                               _I64, _P, _P]
        L.oracle_sparse_attention.argtypes = [_P, _P, _P, _I64, _I64, _I, _P, _P,
                                              _D, _P, _I64, _P, _P]
    return _lib


def num_threads() -> int:
    return lib().oracle_num_threads()


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def as_u16(x) -> np.ndarray:
    """bf16 torch tensor (or uint16 array) -> contiguous uint16 numpy view."""
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.uint16)
    import torch
    assert x.dtype == torch.bfloat16
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_bf16_tensor(u16: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def fractal_order(T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    out = np.empty(T * H * W, dtype=np.int64)
    lib().oracle_fractal_order(T, H, W, P, _ptr(out))
    return out


def flatten(x, T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    """x: [..., N, d] bf16 (raster) -> uint16 array, same shape, flattened order."""
    a = as_u16(x)
    N, d = a.shape[-2], a.shape[-1]
    assert N == T * H * W
    out = np.empty_like(a)
    lib().oracle_flatten(_ptr(a), _ptr(out), a.size // (N * d), T, H, W, P, d)
    return out


def unflatten(y, T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    a = as_u16(y)
    N, d = a.shape[-2], a.shape[-1]
    out = np.empty_like(a)
    lib().oracle_unflatten(_ptr(a), _ptr(out), a.size // (N * d), T, H, W, P, d)
    return out


def unflatten_f64(y: np.ndarray, T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    a = np.ascontiguousarray(y, dtype=np.float64)
    N, d = a.shape[-2], a.shape[-1]
    out = np.empty_like(a)
    lib().oracle_unflatten_f64(_ptr(a), _ptr(out), a.size // (N * d), T, H, W, P, d)
    return out


def pool(xf, S: int = 64) -> np.ndarray:
    """xf: [..., N, d] bf16 flattened -> fp64 [..., N/S, d] block means."""
    a = as_u16(xf)
    N, d = a.shape[-2], a.shape[-1]
    out = np.empty(a.shape[:-2] + (N // S, d), dtype=np.float64)
    lib().oracle_pool(_ptr(a), _ptr(out), a.size // (N * d), N, d, S)
    return out


def reduced_attention(qp: np.ndarray, kp: np.ndarray, rows=None) -> np.ndarray:
    """Rows of softmax(qp kp^T / sqrt d) per head.  qp, kp: [BH, Nb, d] fp64."""
    qp = np.ascontiguousarray(qp, dtype=np.float64)
    kp = np.ascontiguousarray(kp, dtype=np.float64)
    Nb, d = qp.shape[-2], qp.shape[-1]
    BH = qp.size // (Nb * d)
    if rows is None:
        out = np.empty((BH * Nb, Nb))
        lib().oracle_reduced_attention(_ptr(qp), _ptr(kp), BH, Nb, d, None, 0, _ptr(out))
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((rows.size, Nb))
        lib().oracle_reduced_attention(_ptr(qp), _ptr(kp), BH, Nb, d, _ptr(rows),
                                       rows.size, _ptr(out))
    return out


def select_row(a: np.ndarray, thr: float):
    """CDF/top-p selection of one probability row -> (keep bool[n], diag[5])."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    keep = np.zeros(a.size, dtype=np.uint8)
    diag = np.zeros(5)
    lib().oracle_select_row(_ptr(a), a.size, float(thr), _ptr(keep), _ptr(diag))
    return keep.astype(bool), diag


def sta_keep(r: int, c: int, Hb: int, Wb: int, rt: int = 1, rh: int = 1, rw: int = 1) -> bool:
    return bool(lib().oracle_sta_keep(r, c, Hb, Wb, rt, rh, rw))


def block_mask(qp: np.ndarray, kp: np.ndarray, Hb: int, Wb: int, thr: float,
               use_sta: bool, sta=(1, 1, 1), rows=None):
    """Kept-block flags (uint8, rows x Nb) and cut diagnostics (rows x 5)."""
    qp = np.ascontiguousarray(qp, dtype=np.float64)
    kp = np.ascontiguousarray(kp, dtype=np.float64)
    Nb, d = qp.shape[-2], qp.shape[-1]
    BH = qp.size // (Nb * d)
    if rows is None:
        n, rp = BH * Nb, None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n, rp = rows.size, _ptr(rows)
    keep = np.zeros((n, Nb), dtype=np.uint8)
    diag = np.zeros((n, 5))
    lib().oracle_block_mask(_ptr(qp), _ptr(kp), BH, Nb, d, Hb, Wb, float(thr),
                            int(bool(use_sta)), int(sta[0]), int(sta[1]), int(sta[2]),
                            rp, n, _ptr(keep), _ptr(diag))
    return keep, diag


def block_mask_topk(qp: np.ndarray, kp: np.ndarray, Hb: int, Wb: int, k: int,
                    use_sta: bool, sta=(1, 1, 1), rows=None):
    """Static-ratio mask: kept flags (uint8, rows x Nb) and, per row, the last
    kept and first dropped probabilities (rows x 2)."""
    qp = np.ascontiguousarray(qp, dtype=np.float64)
    kp = np.ascontiguousarray(kp, dtype=np.float64)
    Nb, d = qp.shape[-2], qp.shape[-1]
    BH = qp.size // (Nb * d)
    if rows is None:
        n, rp = BH * Nb, None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n, rp = rows.size, _ptr(rows)
    keep = np.zeros((n, Nb), dtype=np.uint8)
    diag = np.zeros((n, 2))
    lib().oracle_block_mask_topk(_ptr(qp), _ptr(kp), BH, Nb, d, Hb, Wb, int(k),
                                 int(bool(use_sta)), int(sta[0]), int(sta[1]), int(sta[2]),
                                 rp, n, _ptr(keep), _ptr(diag))
    return keep, diag


def select_topk_row(a: np.ndarray, k: int):
    a = np.ascontiguousarray(a, dtype=np.float64)
    keep = np.zeros(a.size, dtype=np.uint8)
    diag = np.zeros(2)
    lib().oracle_select_topk_row(_ptr(a), a.size, int(k), _ptr(keep), _ptr(diag))
    return keep, diag


def sta_mask(T: int, Hb: int, Wb: int, sta=(1, 1, 1)) -> np.ndarray:
    """The STA window alone: kept flags of one head's (T*Hb*Wb)^2 block grid."""
    Nb = T * Hb * Wb
    keep = np.zeros((Nb, Nb), dtype=np.uint8)
    lib().oracle_sta_mask(Nb, Hb, Wb, int(sta[0]), int(sta[1]), int(sta[2]), _ptr(keep))
    return keep


def ambiguous_topk(diag: np.ndarray, eps: float = 1e-5, row_max=None) -> np.ndarray:
    """Static-ratio rows whose kept set is not fixed by fp32-accurate
    probabilities: the last kept and first dropped probabilities within a
    relative eps of each other (a near tie across the cut), or, when the row
    maxima are given, a cut probability below 2^-120 of the row maximum (where
    fp32 storage of the ratio underflows)."""
    last, nxt = diag[:, 0], diag[:, 1]
    amb = (nxt >= 0) & (np.abs(last - nxt) <= eps * np.maximum(last, 1e-300))
    if row_max is not None:
        amb |= (nxt >= 0) & (last < row_max * 2.0 ** -120)
    return amb


# ---------------------------------------------------------------- semantic permutation
def kmeans_init(x_u16: np.ndarray, C: int) -> np.ndarray:
    """Initial centroids of one (batch, head): the tokens at floor(j*N/C)."""
    x = to_f64(x_u16)
    N = x.shape[0]
    return x[(np.arange(C) * N) // C].astype(np.float32)


def to_f64(x_u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    return (np.ascontiguousarray(x_u16, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)


def kmeans_assign(x_u16: np.ndarray, cent: np.ndarray):
    """Labels (int32 [N]) and (best, second) distances for one (b, h)."""
    x = np.ascontiguousarray(x_u16, dtype=np.uint16)
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    N, d = x.shape
    C = cent.shape[0]
    label = np.zeros(N, dtype=np.int32)
    diag = np.zeros((N, 2))
    lib().oracle_kmeans_assign(_ptr(x), _ptr(cent), N, d, C, _ptr(label), _ptr(diag))
    return label, diag


def kmeans_update(x_u16: np.ndarray, label: np.ndarray, cent: np.ndarray):
    """New centroids (member means; empty clusters keep theirs) and sizes."""
    x = np.ascontiguousarray(x_u16, dtype=np.uint16)
    out = np.array(cent, dtype=np.float32, copy=True)
    N, d = x.shape
    C = out.shape[0]
    count = np.zeros(C, dtype=np.int32)
    lib().oracle_kmeans_update(_ptr(x), _ptr(np.ascontiguousarray(label, dtype=np.int32)), N, d,
                               C, _ptr(out), _ptr(count))
    return out, count


def kmeans(x_u16: np.ndarray, C: int, iters: int, init=None):
    """Lloyd's iterations: init -> (assign, update) x iters -> final labels.
    Returns (labels, centroids, sizes)."""
    cent = kmeans_init(x_u16, C) if init is None else np.array(init, dtype=np.float32)
    for _ in range(iters):
        label, _ = kmeans_assign(x_u16, cent)
        cent, count = kmeans_update(x_u16, label, cent)
    label, _ = kmeans_assign(x_u16, cent)
    _, count = kmeans_update(x_u16, label, cent)
    return label, cent, count


def cluster_order(label: np.ndarray, C: int):
    """Stable sort by label: (order int64 [N], start int64 [C+1])."""
    label = np.ascontiguousarray(label, dtype=np.int32)
    order = np.zeros(label.size, dtype=np.int64)
    start = np.zeros(C + 1, dtype=np.int64)
    lib().oracle_cluster_order(_ptr(label), label.size, C, _ptr(order), _ptr(start))
    return order, start


def centroid_topp(cq: np.ndarray, ck: np.ndarray, nk: np.ndarray, p: float):
    """Kept key clusters per query cluster (uint8 [Cq, Ck]) and diagnostics."""
    cq = np.ascontiguousarray(cq, dtype=np.float32)
    ck = np.ascontiguousarray(ck, dtype=np.float32)
    nk = np.ascontiguousarray(nk, dtype=np.int32)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    keep = np.zeros((Cq, Ck), dtype=np.uint8)
    diag = np.zeros((Cq, 5))
    lib().oracle_centroid_topp(_ptr(cq), _ptr(ck), _ptr(nk), Cq, Ck, d, float(p), _ptr(keep),
                               _ptr(diag))
    return keep, diag


def cluster_attention(q_u16, k_u16, v_u16, lq, lk, keep, qtok, scale=None):
    """O (fp64 [len(qtok), d]) and LSE of the listed query tokens of one
    (b, h) over the keys of their kept clusters, original token order."""
    q, k, v = (np.ascontiguousarray(x, dtype=np.uint16) for x in (q_u16, k_u16, v_u16))
    N, d = q.shape
    qtok = np.ascontiguousarray(qtok, dtype=np.int64)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((qtok.size, d))
    lse = np.zeros(qtok.size)
    lib().oracle_cluster_attention(_ptr(q), _ptr(k), _ptr(v), N, d,
                                   _ptr(np.ascontiguousarray(lq, dtype=np.int32)),
                                   _ptr(np.ascontiguousarray(lk, dtype=np.int32)), _ptr(keep),
                                   keep.shape[1], float(scale), _ptr(qtok), qtok.size, _ptr(o),
                                   _ptr(lse))
    return o, lse


def mask_to_csr(keep: np.ndarray):
    """Kept flags (rows x Nb) -> (row_ptr int64, col_idx int32), ascending columns."""
    keep = np.asarray(keep, dtype=bool)
    counts = keep.sum(axis=1)
    row_ptr = np.zeros(keep.shape[0] + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col_idx = np.nonzero(keep)[1].astype(np.int32)
    return row_ptr, col_idx


def sparse_attention(qf, kf, vf, row_ptr, col_idx, scale=None, qblocks=None):
    """Block-sparse attention of flattened bf16 q, k, v ([BH, N, d]).

    Returns (O fp64 [nq*64, d], LSE fp64 [nq*64]) for the listed global query
    blocks (default: all, in order).
    """
    q, k, v = as_u16(qf), as_u16(kf), as_u16(vf)
    N, d = q.shape[-2], q.shape[-1]
    BH = q.size // (N * d)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    if qblocks is None:
        nq, qp = BH * (N // 64), None
    else:
        qblocks = np.ascontiguousarray(qblocks, dtype=np.int64)
        nq, qp = qblocks.size, _ptr(qblocks)
    o = np.empty((nq * 64, d))
    lse = np.empty(nq * 64)
    lib().oracle_sparse_attention(_ptr(q), _ptr(k), _ptr(v), BH, N, d, _ptr(row_ptr),
                                  _ptr(col_idx), float(scale), qp, nq, _ptr(o), _ptr(lse))
    return o, lse


def boundary_rows(diag: np.ndarray, thr: float, eps: float = 1e-5) -> np.ndarray:
    """Rows whose boundary block's cumulative mass lies within eps of 1 - thr:
    the kept prefix mass, or that mass without its last block.  These are the
    only rows on which a kept set computed from probabilities accurate to a
    few 1e-7 may legitimately differ from the exact one; every other row,
    near ties across the cut included, has one kept set.  thr = 0 keeps every
    block: never a boundary row."""
    if thr <= 0.0:
        return np.zeros(diag.shape[0], dtype=bool)
    tgt = 1.0 - thr
    return (np.abs(diag[:, 0] - tgt) <= eps) | (np.abs(tgt - diag[:, 1]) <= eps)


def near_tie_rows(diag: np.ndarray, thr: float, eps: float = 1e-5) -> np.ndarray:
    """Rows whose last kept and first dropped blocks have probabilities within
    a relative eps of each other (a near tie across the cut)."""
    if thr <= 0.0:
        return np.zeros(diag.shape[0], dtype=bool)
    dropped = diag[:, 3] >= 0
    return dropped & (diag[:, 2] - diag[:, 3] <= eps * diag[:, 2])


def ambiguous_rows(diag: np.ndarray, thr: float, eps: float = 1e-5) -> np.ndarray:
    """Rows whose CDF cut is numerically ambiguous.

    A row is ambiguous when the kept prefix mass, or that mass without its last
    block, lies within eps of 1 - thr, or when the last kept and first dropped
    blocks have probabilities within a relative eps of each other (a near tie
    across the cut).  Under any per-probability error well below eps, all other
    rows have a unique kept set.  thr = 0 keeps every block: never ambiguous.
    """
    if thr <= 0.0:
        return np.zeros(diag.shape[0], dtype=bool)
    tgt = 1.0 - thr
    near_mass = (np.abs(diag[:, 0] - tgt) <= eps) | (np.abs(tgt - diag[:, 1]) <= eps)
    dropped = diag[:, 3] >= 0
    near_tie = dropped & (diag[:, 2] - diag[:, 3] <= eps * diag[:, 2])
    return near_mass | near_tie
