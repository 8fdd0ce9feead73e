"""Content-adaptive block-sparse video attention on B200 (sm_100a).

Python face of libvsa.  Each function passes device pointers of torch CUDA
tensors and the current CUDA stream to the C ABI (include/vsa.h); torch is
used for device memory and streams only.  Steps (NABLA, Methodology 1-3):

    fractal_flatten -> pool_qk -> block_mask -> sparse_attn_fwd -> fractal_unflatten

`attention_layer` chains the middle three for one attention layer.
"""
from __future__ import annotations

import dataclasses
import math

import torch

from . import _lib
from ._lib import VsaError, vsa_mask_params, vsa_shape

__all__ = ["Shape", "MaskParams", "VsaError", "fractal_flatten", "fractal_unflatten",
           "flatten_pool_qk", "pool_qk_raster", "sparse_attn_fwd_raster",
           "sparse_attn_fwd_to_raster", "Layer",
           "pool_qk", "block_mask", "block_mask_topk", "sta_mask", "sta_mask_nnz",
           "block_mask_workspace_size", "sparse_attn_fwd", "sparse_attn_fwd_rows",
           "ClusterParams", "cluster_attention", "cluster_attn_workspace_size",
           "sparse_attn_workspace_size", "attention_layer", "device_status", "version",
           "Csr"]


@dataclasses.dataclass(frozen=True)
class Shape:
    B: int
    heads: int
    T: int
    H: int
    W: int
    d: int
    P: int = 8

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def Nb(self) -> int:
        return self.N // 64

    def c(self) -> vsa_shape:
        return vsa_shape(self.B, self.heads, self.T, self.H, self.W, self.d, self.P)

    @staticmethod
    def of(wl) -> "Shape":
        return Shape(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, wl.P)


@dataclasses.dataclass(frozen=True)
class MaskParams:
    thr: float
    use_sta: bool = False
    sta: tuple = (1, 1, 1)

    def c(self) -> vsa_mask_params:
        return vsa_mask_params(float(self.thr), int(bool(self.use_sta)), *map(int, self.sta))


@dataclasses.dataclass
class Csr:
    row_ptr: torch.Tensor      # int64 [B*heads*Nb + 1]
    col_idx: torch.Tensor      # int32 [capacity]; entries [0, row_ptr[-1]) are valid
    kept_count: torch.Tensor   # int32 [B*heads*Nb]


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes_void(s.cuda_stream)


def ctypes_void(v):
    import ctypes
    return ctypes.c_void_p(v)


def _ptr(t: torch.Tensor):
    assert t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return ctypes_void(t.data_ptr())


def version() -> str:
    return _lib.load().vsa_version().decode()


def fractal_flatten(x: torch.Tensor, shape: Shape, out: torch.Tensor | None = None, stream=None):
    """Raster [B,h,N,d] bf16 -> fractal order (each 8x8 patch contiguous)."""
    y = torch.empty_like(x) if out is None else out
    _lib.check(_lib.load().vsa_fractal_flatten(_ptr(x), _ptr(y), shape.c(), _stream(stream)))
    return y


def fractal_unflatten(y: torch.Tensor, shape: Shape, out: torch.Tensor | None = None, stream=None):
    x = torch.empty_like(y) if out is None else out
    _lib.check(_lib.load().vsa_fractal_unflatten(_ptr(y), _ptr(x), shape.c(), _stream(stream)))
    return x


def pool_qk(qf: torch.Tensor, kf: torch.Tensor, shape: Shape, out=None, stream=None):
    """64-token block means of Q and K -> (qp, kp) fp64 [B,h,Nb,d]."""
    if out is None:
        sz = (shape.B, shape.heads, shape.Nb, shape.d)
        out = (torch.empty(sz, dtype=torch.float64, device=qf.device),
               torch.empty(sz, dtype=torch.float64, device=qf.device))
    qp, kp = out
    _lib.check(_lib.load().vsa_pool_qk(_ptr(qf), _ptr(kf), _ptr(qp), _ptr(kp), shape.c(),
                                       _stream(stream)))
    return qp, kp


def flatten_pool_qk(q: torch.Tensor, k: torch.Tensor, shape: Shape, out=None, stream=None):
    """Fractal flatten of raster Q and K plus their 64-token block means in one
    pass -> (qf, kf, qp, kp); identical to fractal_flatten + pool_qk."""
    if out is None:
        sz = (shape.B, shape.heads, shape.Nb, shape.d)
        out = (torch.empty_like(q), torch.empty_like(k),
               torch.empty(sz, dtype=torch.float64, device=q.device),
               torch.empty(sz, dtype=torch.float64, device=q.device))
    qf, kf, qp, kp = out
    _lib.check(_lib.load().vsa_flatten_pool_qk(_ptr(q), _ptr(k), _ptr(qf), _ptr(kf), _ptr(qp),
                                               _ptr(kp), shape.c(), _stream(stream)))
    return qf, kf, qp, kp


def pool_qk_raster(q: torch.Tensor, k: torch.Tensor, shape: Shape, out=None, stream=None):
    """64-token block means of the fractal blocks read straight from raster Q
    and K -> (qp, kp); identical to the means of flatten_pool_qk, with no
    flattened copy written."""
    if out is None:
        sz = (shape.B, shape.heads, shape.Nb, shape.d)
        out = (torch.empty(sz, dtype=torch.float64, device=q.device),
               torch.empty(sz, dtype=torch.float64, device=q.device))
    qp, kp = out
    _lib.check(_lib.load().vsa_pool_qk_raster(_ptr(q), _ptr(k), _ptr(qp), _ptr(kp), shape.c(),
                                              _stream(stream)))
    return qp, kp


def block_mask_workspace_size(shape: Shape) -> int:
    return int(_lib.load().vsa_block_mask_workspace_size(shape.c()))


def sparse_attn_workspace_size(shape: Shape) -> int:
    return int(_lib.load().vsa_sparse_attn_workspace_size(shape.c()))


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def block_mask(qp: torch.Tensor, kp: torch.Tensor, shape: Shape, params: MaskParams,
               out: Csr | None = None, workspace: torch.Tensor | None = None, stream=None) -> Csr:
    """Per-row CDF (top-p) block selection [+ STA union] -> CSR kept lists."""
    rows = shape.B * shape.heads * shape.Nb
    dev = qp.device
    if out is None:
        out = Csr(torch.empty(rows + 1, dtype=torch.int64, device=dev),
                  torch.empty(max(rows * shape.Nb, 1), dtype=torch.int32, device=dev),
                  torch.empty(max(rows, 1), dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = _workspace(block_mask_workspace_size(shape), dev)
    _lib.check(_lib.load().vsa_block_mask(
        _ptr(qp), _ptr(kp), shape.c(), params.c(), _ptr(out.row_ptr), _ptr(out.col_idx),
        out.col_idx.numel(), _ptr(out.kept_count), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out


def block_mask_topk(qp: torch.Tensor, kp: torch.Tensor, shape: Shape, k: int,
                    params: MaskParams | None = None, out: Csr | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> Csr:
    """Static-ratio selection: each row's k most probable blocks [+ STA union
    from params; params.thr is ignored] -> CSR kept lists."""
    params = MaskParams(0.0, False) if params is None else params
    rows = shape.B * shape.heads * shape.Nb
    dev = qp.device
    if out is None:
        out = Csr(torch.empty(rows + 1, dtype=torch.int64, device=dev),
                  torch.empty(max(rows * shape.Nb, 1), dtype=torch.int32, device=dev),
                  torch.empty(max(rows, 1), dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = _workspace(block_mask_workspace_size(shape), dev)
    _lib.check(_lib.load().vsa_block_mask_topk(
        _ptr(qp), _ptr(kp), shape.c(), int(k), params.c(), _ptr(out.row_ptr),
        _ptr(out.col_idx), out.col_idx.numel(), _ptr(out.kept_count), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return out


def sta_mask_nnz(shape: Shape, radii=(1, 1, 1)) -> int:
    """Entries of the STA-only mask: heads x product of summed clipped widths."""
    def total(n, r):
        return sum(min(c + r, n - 1) - max(c - r, 0) + 1 for c in range(n))
    Hb, Wb = shape.H // shape.P, shape.W // shape.P
    return (shape.B * shape.heads * total(shape.T, radii[0]) * total(Hb, radii[1])
            * total(Wb, radii[2]))


def sta_mask(shape: Shape, radii=(1, 1, 1), out: Csr | None = None, device="cuda",
             stream=None) -> Csr:
    """The STA window alone as the block mask (no pooling, no scores)."""
    rows = shape.B * shape.heads * shape.Nb
    if out is None:
        nnz = sta_mask_nnz(shape, radii)
        out = Csr(torch.empty(rows + 1, dtype=torch.int64, device=device),
                  torch.empty(max(nnz, 1), dtype=torch.int32, device=device),
                  torch.empty(max(rows, 1), dtype=torch.int32, device=device))
    _lib.check(_lib.load().vsa_sta_mask(
        shape.c(), int(radii[0]), int(radii[1]), int(radii[2]), _ptr(out.row_ptr),
        _ptr(out.col_idx), out.col_idx.numel(), _ptr(out.kept_count), _stream(stream)))
    return out


def sparse_attn_fwd(qf, kf, vf, row_ptr, col_idx, shape: Shape, scale: float = 0.0,
                    out=None, workspace=None, stream=None):
    """Block-sparse attention over the kept 64x64 tiles -> (o bf16, lse fp32)."""
    if out is None:
        out = (torch.empty_like(qf),
               torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=qf.device))
    o, lse = out
    if workspace is None:
        workspace = _workspace(sparse_attn_workspace_size(shape), qf.device)
    _lib.check(_lib.load().vsa_sparse_attn_fwd(
        _ptr(qf), _ptr(kf), _ptr(vf), _ptr(row_ptr), _ptr(col_idx), shape.c(), float(scale),
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def sparse_attn_fwd_raster(q, k, v, row_ptr, col_idx, shape: Shape, scale: float = 0.0,
                           out=None, workspace=None, stream=None):
    """sparse_attn_fwd on raster-order q, k, v -> raster-order (o, lse); the
    mask still indexes fractal blocks.  Equals flattening, sparse_attn_fwd and
    unflattening, bit for bit, without the permuted copies."""
    if out is None:
        out = (torch.empty_like(q),
               torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=q.device))
    o, lse = out
    if workspace is None:
        workspace = _workspace(sparse_attn_workspace_size(shape), q.device)
    _lib.check(_lib.load().vsa_sparse_attn_fwd_raster(
        _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col_idx), shape.c(), float(scale),
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def sparse_attn_fwd_to_raster(qf, kf, vf, row_ptr, col_idx, shape: Shape, scale: float = 0.0,
                              out=None, workspace=None, stream=None):
    """sparse_attn_fwd on flattened qf, kf, vf -> raster-order (o, lse): the
    output unflattening done by the attention's stores.  Equals sparse_attn_fwd
    followed by fractal_unflatten of o (and the same permutation of lse), bit
    for bit."""
    if out is None:
        out = (torch.empty_like(qf),
               torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=qf.device))
    o, lse = out
    if workspace is None:
        workspace = _workspace(sparse_attn_workspace_size(shape), qf.device)
    _lib.check(_lib.load().vsa_sparse_attn_fwd_to_raster(
        _ptr(qf), _ptr(kf), _ptr(vf), _ptr(row_ptr), _ptr(col_idx), shape.c(), float(scale),
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def sparse_attn_fwd_rows(qf, kf, vf, row_ptr, col_idx, shape: Shape, qblocks: torch.Tensor,
                         scale: float = 0.0, out=None, workspace=None, stream=None):
    """Attention for the listed query blocks only (int32 global block rows,
    strictly ascending); other rows of `out` are left as they are."""
    if out is None:
        out = (torch.zeros_like(qf),
               torch.full((shape.B, shape.heads, shape.N), float("nan"), dtype=torch.float32,
                          device=qf.device))
    o, lse = out
    if workspace is None:
        workspace = _workspace(sparse_attn_workspace_size(shape), qf.device)
    qb = qblocks.to(device=qf.device, dtype=torch.int32).contiguous()
    _lib.check(_lib.load().vsa_sparse_attn_fwd_rows(
        _ptr(qf), _ptr(kf), _ptr(vf), _ptr(row_ptr), _ptr(col_idx), shape.c(), float(scale),
        _ptr(qb) if qb.numel() else ctypes_void(0), qb.numel(), _ptr(o), _ptr(lse),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


@dataclasses.dataclass
class ClusterParams:
    """Semantic-aware permutation: clusters of Q and K, Lloyd iterations, and
    the estimated-attention mass kept per query cluster."""
    Cq: int = 256
    Ck: int = 512
    iters: int = 2
    p: float = 0.9

    def c(self):
        return _lib.vsa_cluster_params(int(self.Cq), int(self.Ck), int(self.iters),
                                       float(self.p))


def cluster_attn_workspace_size(shape: Shape, params: ClusterParams) -> int:
    return int(_lib.load().vsa_cluster_attn_workspace_size(shape.c(), params.c()))


def cluster_attention(q, k, v, shape: Shape, params: ClusterParams, scale: float = 0.0,
                      init=None, want_state: bool = False, out=None, workspace=None,
                      stream=None):
    """k-means permutation + centroid top-p + attention over the kept clusters
    -> (o, lse) in the input token order, plus the intermediate state (labels,
    sizes, centroids, kept flags) when want_state is set.  `init` is an
    optional (q_centroids, k_centroids) pair of fp32 [B,h,C,d] tensors."""
    import ctypes
    dev = q.device
    if out is None:
        out = (torch.empty_like(q),
               torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=dev))
    o, lse = out
    if workspace is None:
        workspace = _workspace(cluster_attn_workspace_size(shape, params), dev)
    B, h, N, d = shape.B, shape.heads, shape.N, shape.d
    st = None
    if want_state:
        i32, f32 = torch.int32, torch.float32
        st = {"q_labels": torch.empty((B, h, N), dtype=i32, device=dev),
              "k_labels": torch.empty((B, h, N), dtype=i32, device=dev),
              "q_counts": torch.empty((B, h, params.Cq), dtype=i32, device=dev),
              "k_counts": torch.empty((B, h, params.Ck), dtype=i32, device=dev),
              "q_centroids": torch.empty((B, h, params.Cq, d), dtype=f32, device=dev),
              "k_centroids": torch.empty((B, h, params.Ck, d), dtype=f32, device=dev),
              "keep": torch.empty((B, h, params.Cq, params.Ck), dtype=torch.uint8, device=dev)}
        cst = _lib.vsa_cluster_state(*(t.data_ptr() for t in st.values()))
        cst_ptr = ctypes.pointer(cst)
    else:
        cst_ptr = None
    iq, ik = (None, None) if init is None else init
    _lib.check(_lib.load().vsa_cluster_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), shape.c(), params.c(), float(scale),
        _ptr(iq) if iq is not None else ctypes_void(0),
        _ptr(ik) if ik is not None else ctypes_void(0), _ptr(o), _ptr(lse), cst_ptr,
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return (o, lse, st) if want_state else (o, lse)


def device_status(stream=None) -> None:
    """Synchronise and raise if a kernel recorded a device-side error."""
    _lib.check(_lib.load().vsa_device_status(_stream(stream)))


class Layer:
    """Preallocated buffers for one attention layer: pool, mask, sparse attention.

    layout "flat": q, k, v, o and lse in fractal-flattened token order;
    "raster": in raster order (the fractal blocks are gathered by the kernels'
    own addressing, so no permuted copy is made)."""

    def __init__(self, shape: Shape, params: MaskParams, device="cuda", scale: float = 0.0,
                 layout: str = "flat"):
        if layout not in ("flat", "raster"):
            raise ValueError(f"layout must be 'flat' or 'raster', not {layout!r}")
        self.shape, self.params, self.scale, self.layout = shape, params, scale, layout
        B, h, Nb, d, N = shape.B, shape.heads, shape.Nb, shape.d, shape.N
        f64 = dict(dtype=torch.float64, device=device)
        self.qp = torch.empty((B, h, Nb, d), **f64)
        self.kp = torch.empty((B, h, Nb, d), **f64)
        rows = B * h * Nb
        self.csr = Csr(torch.empty(rows + 1, dtype=torch.int64, device=device),
                       torch.empty(max(rows * Nb, 1), dtype=torch.int32, device=device),
                       torch.empty(max(rows, 1), dtype=torch.int32, device=device))
        self.ws_mask = _workspace(block_mask_workspace_size(shape), device)
        self.ws_attn = _workspace(sparse_attn_workspace_size(shape), device)
        self.o = torch.empty((B, h, N, d), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((B, h, N), dtype=torch.float32, device=device)

    def __call__(self, q, k, v, stream=None):
        raster = self.layout == "raster"
        (pool_qk_raster if raster else pool_qk)(q, k, self.shape, out=(self.qp, self.kp),
                                                stream=stream)
        block_mask(self.qp, self.kp, self.shape, self.params, out=self.csr,
                   workspace=self.ws_mask, stream=stream)
        (sparse_attn_fwd_raster if raster else sparse_attn_fwd)(
            q, k, v, self.csr.row_ptr, self.csr.col_idx, self.shape, self.scale,
            out=(self.o, self.lse), workspace=self.ws_attn, stream=stream)
        return self.o, self.lse


def attention_layer(qf, kf, vf, shape: Shape, params: MaskParams, scale: float = 0.0):
    """pool -> mask -> sparse attention on flattened bf16 q, k, v (allocating)."""
    return Layer(shape, params, qf.device, scale)(qf, kf, vf)
