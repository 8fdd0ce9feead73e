"""The seeded input generator: deterministic, shaped as stated, heads independent."""
import numpy as np
import torch

from content_adaptive_block_fractal_b200 import workloads


def test_config_shapes():
    sizes = {"tiny": (2, 64, 1024, 16), "wan1.3b-480p": (12, 128, 32256, 504),
             "wan14b-720p": (40, 128, 80640, 1260), "long-241f": (24, 128, 234240, 3660)}
    for name, (h, d, N, Nb) in sizes.items():
        wl = workloads.get(name)
        assert (wl.heads, wl.d, wl.N, wl.Nb) == (h, d, N, Nb)
    assert len(workloads.sweep_workloads()) == 10


def test_deterministic_and_head_independent():
    wl = workloads.get("tiny")
    q1, k1, v1 = workloads.make_qkv(wl)
    q2, k2, v2 = workloads.make_qkv(wl)
    assert q1.dtype == torch.bfloat16 and q1.shape == (1, 2, 1024, 64)
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    qh, _, _ = workloads.make_qkv(wl, heads=[1])
    assert torch.equal(qh[0, 0], q1[0, 1])


def test_labels_cover_clusters_and_drift():
    wl = workloads.get("wan1.3b-480p")
    lab = workloads.labels(wl)
    assert lab.shape == (wl.T, wl.H, wl.W)
    assert lab.min() >= 0 and lab.max() < wl.clusters
    assert len(np.unique(lab)) > wl.clusters // 2
    assert (lab[0] != lab[-1]).any()          # Voronoi cells move over time


def test_cluster_structure_visible_in_qk():
    wl = workloads.get("tiny")
    q, k, _ = workloads.make_qkv(wl)
    lab = workloads.labels(wl).reshape(-1)
    qd, kd = q[0, 0].double(), k[0, 0].double()
    same = lab[:, None] == lab[None, :]
    s = (qd[:200] @ kd.T).numpy()
    assert s[same[:200]].mean() > s[~same[:200]].mean() + 50.0


def test_random_csr_is_valid():
    rp, ci = workloads.random_csr(50, 16, 0.2, seed=3)
    assert rp[0] == 0 and rp[-1] == ci.size and (np.diff(rp) >= 1).all()
    for r in range(50):
        row = ci[rp[r]:rp[r + 1]]
        assert (np.diff(row) > 0).all() and row.min() >= 0 and row.max() < 16
