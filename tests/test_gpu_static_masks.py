"""GPU parity of the static-ratio (top-k) selection and of the STA window used
as the whole mask, against the oracle; and attention on those masks."""
import functools

import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3
AMBIG_EPS = 1e-5


@functools.lru_cache(maxsize=4)
def pooled(name):
    wl = workloads.get(name)
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    return wl, (qf, kf, vf), oracle.pool(qf), oracle.pool(kf)


def dev(x):
    if x.dtype == np.uint16:
        return oracle.to_bf16_tensor(x).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def csr_rows(csr):
    rp = csr.row_ptr.cpu().numpy()
    ci = csr.col_idx.cpu().numpy()
    return rp, ci


def check_structure(csr, rows, Nb):
    rp, ci = csr_rows(csr)
    cnt = csr.kept_count.cpu().numpy()[:rows]
    assert rp[0] == 0 and np.array_equal(np.diff(rp), cnt)
    return rp, ci


def row_max_prob(qp, kp, rows=None):
    """Largest reduced-attention probability of each row (for the underflow
    part of the ambiguity rule)."""
    a = oracle.reduced_attention(qp, kp, rows)
    return a.max(axis=1)


# ---------------------------------------------------------------- f3 STA window alone
@pytest.mark.parametrize("T,H,W,heads,rad", [
    (4, 16, 16, 2, (1, 1, 1)), (3, 16, 24, 3, (0, 0, 0)), (5, 24, 16, 1, (2, 1, 1)),
    (2, 8, 8, 2, (9, 9, 9)), (21, 32, 48, 2, (1, 1, 1)), (6, 16, 40, 2, (1, 0, 3)),
])
def test_sta_mask_matches_oracle(T, H, W, heads, rad):
    shape = vsa.Shape(1, heads, T, H, W, 64)
    csr = vsa.sta_mask(shape, rad)
    Nb, Hb, Wb = shape.Nb, H // 8, W // 8
    rp, ci = check_structure(csr, heads * Nb, Nb)
    keep = oracle.sta_mask(T, Hb, Wb, rad)
    rp_o, ci_o = oracle.mask_to_csr(np.tile(keep, (heads, 1)))
    np.testing.assert_array_equal(rp, rp_o)
    np.testing.assert_array_equal(ci[:rp[-1]], ci_o)
    assert rp[-1] == vsa.sta_mask_nnz(shape, rad)
    vsa.device_status()


def test_attention_on_sta_mask():
    wl, (qf, kf, vf), _, _ = pooled("wan1.3b-480p")
    shape = vsa.Shape.of(wl)
    csr = vsa.sta_mask(shape, (1, 1, 1))
    o, lse = vsa.sparse_attn_fwd(dev(qf), dev(kf), dev(vf), csr.row_ptr, csr.col_idx, shape)
    rp, ci = csr_rows(csr)
    qb = np.sort(np.random.default_rng(3).choice(wl.heads * wl.Nb, 40, replace=False))
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci[:rp[-1]], qblocks=qb)
    og = o.reshape(-1, 64, wl.d)[torch.as_tensor(qb).cuda()].float().cpu().numpy()
    lg = lse.reshape(-1, 64)[torch.as_tensor(qb).cuda()].cpu().numpy()
    err = np.abs(og.reshape(o_ref.shape) - o_ref)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    assert np.abs(lg.reshape(-1) - lse_ref).max() <= LSE_TOL
    vsa.device_status()


# ---------------------------------------------------------------- f2 static ratio
def compare_topk(csr, keep_o, diag_o, rowmax, rows_idx=None):
    rp, ci = csr_rows(csr)
    amb = oracle.ambiguous_topk(diag_o, AMBIG_EPS, rowmax)
    rows_idx = np.arange(keep_o.shape[0]) if rows_idx is None else rows_idx
    n_amb = bad_amb = 0
    for i, g in enumerate(rows_idx):
        got = ci[rp[g]:rp[g + 1]]
        want = np.nonzero(keep_o[i])[0]
        if amb[i]:
            n_amb += 1
            bad_amb += not np.array_equal(got, want)
            continue
        np.testing.assert_array_equal(got, want, err_msg=f"row {g}")
    return n_amb, bad_amb


@pytest.mark.parametrize("name", ["tiny", "wan1.3b-480p"])
@pytest.mark.parametrize("frac,sta", [(0.0, False), (0.1, False), (0.1, True), (0.3, True),
                                      (0.999, False), (1.0, False), (2.0, True)])
def test_topk_matches_oracle(name, frac, sta):
    wl, _, qp, kp = pooled(name)
    shape = vsa.Shape.of(wl)
    k = max(1, int(round(frac * wl.Nb)))
    params = vsa.MaskParams(0.0, sta)
    csr = vsa.block_mask_topk(dev(qp), dev(kp), shape, k, params)
    check_structure(csr, wl.heads * wl.Nb, wl.Nb)
    keep, diag = oracle.block_mask_topk(qp, kp, wl.Hb, wl.Wb, k, sta)
    n_amb, bad = compare_topk(csr, keep, diag, row_max_prob(qp, kp))
    print(f"\n{name} k={k} sta={sta}: {n_amb} rows near the cut, {bad} differ")
    if not sta:
        cnt = csr.kept_count.cpu().numpy()[:wl.heads * wl.Nb]
        assert (cnt == min(k, wl.Nb)).all()
    vsa.device_status()


def test_topk_exact_ties_go_to_lower_index():
    """Duplicated key blocks give exactly equal probabilities; with Nb <= 128
    they share a score tile, so the GPU sees them equal too, and the cut must
    take them in index order in every row."""
    wl, _, qp, kp = pooled("tiny")
    kp2 = kp.copy()
    kp2[..., 1::2, :] = kp2[..., 0::2, :]          # blocks 2i and 2i+1 identical
    shape = vsa.Shape.of(wl)
    for k in (1, 2, 3, 5, 8, 15):
        csr = vsa.block_mask_topk(dev(qp), dev(kp2), shape, k)
        keep, diag = oracle.block_mask_topk(qp, kp2, wl.Hb, wl.Wb, k, False)
        rp, ci = csr_rows(csr)
        for g in range(keep.shape[0]):
            np.testing.assert_array_equal(ci[rp[g]:rp[g + 1]], np.nonzero(keep[g])[0],
                                          err_msg=f"k={k} row {g}")


def test_attention_on_topk_mask():
    wl, (qf, kf, vf), qp, kp = pooled("wan1.3b-480p")
    shape = vsa.Shape.of(wl)
    csr = vsa.block_mask_topk(dev(qp), dev(kp), shape, wl.Nb // 10, vsa.MaskParams(0.0, True))
    o, lse = vsa.sparse_attn_fwd(dev(qf), dev(kf), dev(vf), csr.row_ptr, csr.col_idx, shape)
    rp, ci = csr_rows(csr)
    qb = np.sort(np.random.default_rng(4).choice(wl.heads * wl.Nb, 40, replace=False))
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci[:rp[-1]], qblocks=qb)
    og = o.reshape(-1, 64, wl.d)[torch.as_tensor(qb).cuda()].float().cpu().numpy()
    lg = lse.reshape(-1, 64)[torch.as_tensor(qb).cuda()].cpu().numpy()
    err = np.abs(og.reshape(o_ref.shape) - o_ref)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    assert np.abs(lg.reshape(-1) - lse_ref).max() <= LSE_TOL
    vsa.device_status()
