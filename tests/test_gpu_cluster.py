"""GPU parity of the semantic-aware permutation path (k-means, permutation,
centroid top-p, attention over kept clusters) against the oracle.

k-means under floating point has one exact answer but is ill-conditioned
(a label decided within rounding changes the next centroids), so every step
is checked on the GPU's own state: the final labels are the argmin for the
GPU's final centroids (except assignments within rounding of a tie), the
sizes are the label counts, the kept clusters are the oracle's top-p on the
GPU's centroids and sizes, and the output is the oracle's attention on the
GPU's labels and kept clusters.  A from-scratch oracle run is also compared
and its agreement reported."""
import functools

import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


@functools.lru_cache(maxsize=4)
def data(name, heads):
    wl = workloads.get(name)
    q, k, v = workloads.make_qkv(wl, heads=range(heads))
    return wl, q, k, v


def check_case(name, heads, params, n_tok=96, init=False):
    wl, q, k, v = data(name, heads)
    shape = vsa.Shape(wl.B, heads, wl.T, wl.H, wl.W, wl.d)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse, st = vsa.cluster_attention(qd, kd, vd, shape, params, want_state=True)
    vsa.device_status()
    st = {key: t.cpu().numpy() for key, t in st.items()}
    rng = np.random.default_rng(21)
    mism = total = 0
    for h in range(heads):
        qu, ku, vu = (oracle.as_u16(x)[0, h] for x in (q, k, v))
        for side, xu, C in (("q", qu, params.Cq), ("k", ku, params.Ck)):
            lab = st[f"{side}_labels"][0, h]
            cent = st[f"{side}_centroids"][0, h]
            cnt = st[f"{side}_counts"][0, h]
            np.testing.assert_array_equal(cnt, np.bincount(lab, minlength=C))
            want, diag = oracle.kmeans_assign(xu, cent)
            gap = (diag[:, 1] - diag[:, 0]) / np.maximum(np.abs(diag[:, 0]), 1.0)
            bad = (lab != want) & (gap > 1e-4)
            assert not bad.any(), f"{side} head {h}: {bad.sum()} labels not the argmin"
            # the whole run from scratch on the CPU
            ref_lab, ref_cent, _ = oracle.kmeans(xu, C, params.iters)
            mism += int((ref_lab != lab).sum())
            total += lab.size
        keep = st["keep"][0, h]
        ref_keep, kdiag = oracle.centroid_topp(st["q_centroids"][0, h], st["k_centroids"][0, h],
                                               st["k_counts"][0, h], params.p)
        amb = oracle.ambiguous_rows(kdiag, 1.0 - float(np.float32(params.p)), 1e-9)
        rows_bad = np.nonzero((keep != ref_keep).any(axis=1) & ~amb)[0]
        assert rows_bad.size == 0, f"head {h}: kept clusters differ in rows {rows_bad[:8]}"
        tok = np.sort(rng.choice(wl.N, n_tok, replace=False))
        o_ref, l_ref = oracle.cluster_attention(qu, ku, vu, st["q_labels"][0, h],
                                                st["k_labels"][0, h], keep, tok)
        og = o[0, h, torch.as_tensor(tok).cuda()].float().cpu().numpy()
        lg = lse[0, h, torch.as_tensor(tok).cuda()].cpu().numpy()
        err = np.abs(og - o_ref)
        print(f"\n{name} h{h} Cq={params.Cq} Ck={params.Ck} it={params.iters} p={params.p}: "
              f"kept {keep.mean():.3f}, O max {err.max():.2e} mean {err.mean():.2e}, "
              f"LSE max {np.abs(lg - l_ref).max():.2e}")
        assert err.max() <= O_MAX and err.mean() <= O_MEAN
        assert np.abs(lg - l_ref).max() <= LSE_TOL
    print(f"labels agreeing with a from-scratch oracle run: {total - mism}/{total}")
    assert mism <= 0.01 * total
    if init:
        # the centroid cache path: the same initial centroids passed in
        ci = [torch.from_numpy(np.stack([oracle.kmeans_init(oracle.as_u16(x)[0, h], C)
                                         for h in range(heads)])[None]).cuda()
              for x, C in ((q, params.Cq), (k, params.Ck))]
        o2, l2 = vsa.cluster_attention(qd, kd, vd, shape, params, init=tuple(ci))
        vsa.device_status()
        assert torch.equal(o2, o) and torch.equal(l2, lse)


@pytest.mark.parametrize("name,heads,params,init", [
    ("tiny", 2, vsa.ClusterParams(8, 16, 2, 0.8), True),
    ("tiny", 2, vsa.ClusterParams(5, 7, 0, 0.5), False),
    ("tiny", 1, vsa.ClusterParams(16, 16, 3, 1.0), False),      # p = 1: every cluster kept
    ("wan1.3b-480p", 2, vsa.ClusterParams(64, 128, 2, 0.9), True),
    ("wan1.3b-480p", 1, vsa.ClusterParams(100, 300, 1, 0.7), False),
])
def test_cluster_attention_matches_oracle(name, heads, params, init):
    check_case(name, heads, params, init=init)


def test_cluster_attention_p1_is_dense():
    wl, q, k, v = data("tiny", 1)
    shape = vsa.Shape(wl.B, 1, wl.T, wl.H, wl.W, wl.d)
    o, lse = vsa.cluster_attention(q.cuda(), k.cuda(), v.cuda(), shape,
                                   vsa.ClusterParams(4, 8, 1, 1.0))
    vsa.device_status()
    qt, kt, vt = (x[0, 0].double() for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    err = (o[0, 0].double().cpu() - ref).abs()
    assert err.max().item() <= O_MAX and err.mean().item() <= O_MEAN


@pytest.mark.parametrize("name,C", [("tiny", 16), ("wan1.3b-480p", 128)])
def test_centroid_update_matches_oracle_on_gpu_labels(name, C):
    """The GPU's centroid update element by element: with the same initial
    centroids, a run without iterations returns the first assignment, and a
    run with one iteration returns the centroids updated from exactly that
    assignment; the oracle's update of the same labels must give the same
    fp32 centroids (fp64 member means of bf16 values, rounded once)."""
    wl, q, k, v = data(name, 1)
    shape = vsa.Shape(wl.B, 1, wl.T, wl.H, wl.W, wl.d)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    qu, ku = (oracle.as_u16(x)[0, 0] for x in (q, k))
    init = [oracle.kmeans_init(xu, C) for xu in (qu, ku)]
    init_d = tuple(torch.from_numpy(c[None, None].copy()).cuda() for c in init)
    _, _, st0 = vsa.cluster_attention(qd, kd, vd, shape, vsa.ClusterParams(C, C, 0, 0.9),
                                      init=init_d, want_state=True)
    _, _, st1 = vsa.cluster_attention(qd, kd, vd, shape, vsa.ClusterParams(C, C, 1, 0.9),
                                      init=init_d, want_state=True)
    vsa.device_status()
    for side, xu, c0 in (("q", qu, init[0]), ("k", ku, init[1])):
        lab0 = st0[f"{side}_labels"][0, 0].cpu().numpy()
        np.testing.assert_array_equal(st0[f"{side}_centroids"][0, 0].cpu().numpy(), c0)
        want, count = oracle.kmeans_update(xu, lab0, c0)
        got = st1[f"{side}_centroids"][0, 0].cpu().numpy()
        ulp = np.spacing(np.abs(want).astype(np.float32))
        assert (np.abs(got - want) <= ulp).all(), f"{side}: max diff {np.abs(got - want).max()}"
        exact = float((got == want).mean())
        print(f"\n{name} {side} C={C}: {exact:.5f} of centroid entries bit-identical")
