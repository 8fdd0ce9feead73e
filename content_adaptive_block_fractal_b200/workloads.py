"""Seeded synthetic video-token workloads.

This module only draws inputs: grid shapes, cluster labels and Q/K/V values in
raster order.  It holds none of the method's arithmetic (no reordering, pooling,
scoring or selection), so both the CUDA path and the CPU oracle can consume
exactly the same bytes.

Recipe (stands in for Wan 2.1 / HunyuanVideo activations, which are not
available): per head, C cluster centroids c_k ~ N(0, 1)^d; every token carries
the label of its nearest Voronoi seed (Euclidean distance in token units);
Q = 1.5 * c_label + 0.5 * N(0, 1), K likewise with independent noise,
V ~ N(0, 1); values are rounded to bf16 (round to nearest even).  The tiny case
uses static 3-D seeds in [0,T) x [0,H) x [0,W); the larger ones use 2-D seeds
in [0,H) x [0,W) that drift with a per-seed velocity drawn uniformly in a disc
of radius 0.5 tokens per frame.  The 14B-shaped case also divides each head's
Q by a temperature tau_h ~ U[0.5, 2] before rounding.

Every head is drawn from its own PCG64 stream keyed by (seed, head), so any
subset of heads can be regenerated without drawing the others.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

__all__ = ["Workload", "CONFIGS", "SWEEP", "get", "labels", "make_qkv",
           "make_head", "sweep_workloads"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    clusters: int
    thr: float
    use_sta: bool
    seed: int
    P: int = 8
    seeds_3d: bool = False      # static 3-D Voronoi seeds (tiny case)
    temperature: bool = False   # per-head Q temperature tau_h ~ U[0.5, 2]
    sta: tuple = (1, 1, 1)      # STA window radii (frames, patch rows, patch cols)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def block(self) -> int:
        return self.P * self.P

    @property
    def Nb(self) -> int:
        return self.N // self.block

    @property
    def Hb(self) -> int:
        return self.H // self.P

    @property
    def Wb(self) -> int:
        return self.W // self.P

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "heads": self.heads,
                "d": self.d, "grid": [self.T, self.H, self.W], "N": self.N,
                "blocks": self.Nb, "thr": self.thr, "sta": self.use_sta,
                "clusters": self.clusters, "seed": self.seed}


CONFIGS = {
    "tiny": Workload("tiny", B=1, heads=2, d=64, T=4, H=16, W=16, clusters=4,
                     thr=0.2, use_sta=False, seed=2026, seeds_3d=True),
    "wan1.3b-480p": Workload("wan1.3b-480p", B=1, heads=12, d=128, T=21, H=32,
                             W=48, clusters=16, thr=0.2, use_sta=True, seed=2027),
    "wan14b-720p": Workload("wan14b-720p", B=1, heads=40, d=128, T=21, H=48,
                            W=80, clusters=16, thr=0.1, use_sta=True, seed=2028,
                            temperature=True),
    "long-241f": Workload("long-241f", B=1, heads=24, d=128, T=61, H=48, W=80,
                          clusters=32, thr=0.1, use_sta=False, seed=2029),
}

# thr x STA grid at the 14B 720p shape (same generator, same seed).
SWEEP = [(thr, sta) for thr in (0.0, 0.05, 0.1, 0.2, 0.3) for sta in (True, False)]


def get(name: str) -> Workload:
    return CONFIGS[name]


def sweep_workloads():
    base = CONFIGS["wan14b-720p"]
    return [base.replace(name=f"wan14b-720p-thr{thr}-{'sta' if sta else 'nosta'}",
                         thr=thr, use_sta=sta) for thr, sta in SWEEP]


def _layout_rng(wl: Workload) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, 0xC0FFEE])))


def _head_rng(wl: Workload, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, b, h])))


def labels(wl: Workload) -> np.ndarray:
    """Cluster label of every token, int32 array of shape (T, H, W) in raster order."""
    rng = _layout_rng(wl)
    C = wl.clusters
    t = np.arange(wl.T, dtype=np.float64)[:, None, None]
    y = np.arange(wl.H, dtype=np.float64)[None, :, None]
    x = np.arange(wl.W, dtype=np.float64)[None, None, :]
    best = np.full((wl.T, wl.H, wl.W), np.inf)
    lab = np.zeros((wl.T, wl.H, wl.W), dtype=np.int32)
    if wl.seeds_3d:
        seeds = rng.uniform(0.0, 1.0, size=(C, 3)) * np.array([wl.T, wl.H, wl.W])
        for k in range(C):
            dist = (t - seeds[k, 0]) ** 2 + (y - seeds[k, 1]) ** 2 + (x - seeds[k, 2]) ** 2
            upd = dist < best
            best = np.where(upd, dist, best)
            lab = np.where(upd, k, lab)
    else:
        seeds = rng.uniform(0.0, 1.0, size=(C, 2)) * np.array([wl.H, wl.W])
        radius = 0.5 * np.sqrt(rng.uniform(0.0, 1.0, size=C))
        angle = rng.uniform(0.0, 2.0 * math.pi, size=C)
        vel = np.stack([radius * np.sin(angle), radius * np.cos(angle)], axis=1)
        for k in range(C):
            sy = seeds[k, 0] + t * vel[k, 0]
            sx = seeds[k, 1] + t * vel[k, 1]
            dist = (y - sy) ** 2 + (x - sx) ** 2
            upd = dist < best
            best = np.where(upd, dist, best)
            lab = np.where(upd, k, lab)
    return lab.astype(np.int32)


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    # torch's float32 -> bfloat16 conversion rounds to nearest even.
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_head(wl: Workload, b: int, h: int, lab: np.ndarray | None = None):
    """(q, k, v) for one (batch, head): bf16 CPU tensors [N, d], raster order."""
    if lab is None:
        lab = labels(wl)
    rng = _head_rng(wl, b, h)
    d, N = wl.d, wl.N
    cent = rng.standard_normal((wl.clusters, d))
    tau = rng.uniform(0.5, 2.0) if wl.temperature else 1.0
    flat = lab.reshape(-1)
    q = 1.5 * cent[flat] + 0.5 * rng.standard_normal((N, d))
    k = 1.5 * cent[flat] + 0.5 * rng.standard_normal((N, d))
    v = rng.standard_normal((N, d))
    if wl.temperature:
        q = q / tau
    return _to_bf16(q), _to_bf16(k), _to_bf16(v)


def make_qkv(wl: Workload, heads=None, batches=None):
    """Q, K, V as bf16 CPU tensors [B', h', N, d] in raster order.

    ``heads``/``batches`` select a subset (defaults: all); the values of a head do
    not depend on which other heads are drawn.
    """
    heads = list(range(wl.heads)) if heads is None else list(heads)
    batches = list(range(wl.B)) if batches is None else list(batches)
    lab = labels(wl)
    shape = (len(batches), len(heads), wl.N, wl.d)
    q = torch.empty(shape, dtype=torch.bfloat16)
    k = torch.empty(shape, dtype=torch.bfloat16)
    v = torch.empty(shape, dtype=torch.bfloat16)
    for i, b in enumerate(batches):
        for j, h in enumerate(heads):
            q[i, j], k[i, j], v[i, j] = make_head(wl, b, h, lab)
    return q, k, v


def random_csr(n_rows: int, nb: int, density: float, seed: int):
    """Seeded random block lists (row_ptr int64, col_idx int32), ascending per row.

    Used to drive the attention step with masks that come from neither side
    under test.  Every row keeps at least one block.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    keep = rng.uniform(size=(n_rows, nb)) < density
    keep[np.arange(n_rows), rng.integers(0, nb, size=n_rows)] = True
    counts = keep.sum(axis=1)
    row_ptr = np.zeros(n_rows + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col_idx = np.nonzero(keep)[1].astype(np.int32)
    return row_ptr, col_idx


def short_csr(n_rows: int, nb: int, k_min: int, k_max: int, seed: int):
    """Seeded random block lists with k_min..k_max distinct blocks per row
    (row_ptr int64, col_idx int32, ascending per row), drawn row by row so
    that wide grids need no n_rows x nb matrix."""
    rng = np.random.Generator(np.random.PCG64(seed))
    counts = rng.integers(k_min, k_max + 1, size=n_rows)
    row_ptr = np.zeros(n_rows + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col_idx = np.empty(int(row_ptr[-1]), dtype=np.int32)
    # k_max draws per row, duplicates replaced until each row has distinct blocks
    draw = rng.integers(0, nb, size=(n_rows, k_max))
    for r in range(n_rows):
        cols = np.unique(draw[r, :counts[r]])
        while cols.size < counts[r]:
            cols = np.unique(np.append(cols, rng.integers(0, nb)))
        col_idx[row_ptr[r]:row_ptr[r + 1]] = cols
    return row_ptr, col_idx
