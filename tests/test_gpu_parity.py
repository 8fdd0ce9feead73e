"""CUDA path vs the CPU oracle, element by element, on seeded synthetic inputs.

Bars: the flatten permutation, pooled means and the CSR kept lists are
bit-exact (CSR rows whose boundary block's cumulative mass lies within 1e-5
of 1 - thr are counted and reported; rows with a near tie across the cut are
counted too but must match); attention output within max |err| <= 2e-2 and mean |err|
<= 2e-3 of the fp64 oracle, LSE within 1e-3.  The oracle never receives a
value produced by the CUDA path: masks for the attention checks come from the
oracle or from a seeded generator.
"""
import functools
import math

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
def qkv(name):
    return workloads.make_qkv(workloads.get(name))


def dev(x):
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            return oracle.to_bf16_tensor(x).cuda()
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return x.contiguous().cuda()


def u16(t):
    return oracle.as_u16(t.cpu())


def thr32(thr):
    """The ABI carries thr as fp32; the oracle takes the same value."""
    return float(np.float32(thr))


def small_shape(T=3, H=16, W=24, d=128, heads=2, B=1):
    return workloads.Workload("grid", B=B, heads=heads, d=d, T=T, H=H, W=W, clusters=4,
                              thr=0.2, use_sta=True, seed=77, seeds_3d=True)


# ---------------------------------------------------------------- a1 flatten
@pytest.mark.parametrize("wl", [workloads.get("tiny"), small_shape(), small_shape(T=1, H=8, W=8, d=64),
                                workloads.get("wan1.3b-480p")], ids=lambda w: f"{w.name}-{w.T}x{w.H}x{w.W}")
def test_flatten_bit_exact(wl):
    q, _, _ = workloads.make_qkv(wl, heads=range(min(wl.heads, 3)))
    shape = vsa.Shape(wl.B, q.shape[1], wl.T, wl.H, wl.W, wl.d)
    qd = dev(q)
    qf = vsa.fractal_flatten(qd, shape)
    np.testing.assert_array_equal(u16(qf), oracle.flatten(q, wl.T, wl.H, wl.W))
    back = vsa.fractal_unflatten(qf, shape)
    assert torch.equal(back, qd)
    vsa.device_status()


# ---------------------------------------------------------------- a2 pool
@pytest.mark.parametrize("name", ["tiny", "wan1.3b-480p"])
def test_pool_bit_exact(name):
    wl = workloads.get(name)
    q, k, _ = qkv(name)
    qf, kf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k))
    shape = vsa.Shape.of(wl)
    qp, kp = vsa.pool_qk(dev(qf), dev(kf), shape)
    np.testing.assert_array_equal(qp.cpu().numpy(), oracle.pool(qf))
    np.testing.assert_array_equal(kp.cpu().numpy(), oracle.pool(kf))


# ---------------------------------------------------------------- a1+a2 fused
@pytest.mark.parametrize("name,d,heads", [("tiny", None, None), ("wan1.3b-480p", None, 3),
                                          ("tiny", 128, None)])
def test_flatten_pool_fused_bit_exact(name, d, heads):
    wl = workloads.get(name)
    if d is not None:
        wl = workloads.Workload(**{**wl.__dict__, "d": d})
    q, k, _ = workloads.make_qkv(wl, heads=range(heads)) if heads else workloads.make_qkv(wl)
    shape = vsa.Shape(wl.B, q.shape[1], wl.T, wl.H, wl.W, wl.d)
    qd, kd = dev(q), dev(k)
    qf, kf, qp, kp = vsa.flatten_pool_qk(qd, kd, shape)
    qf_o, kf_o = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k))
    np.testing.assert_array_equal(u16(qf), qf_o)
    np.testing.assert_array_equal(u16(kf), kf_o)
    np.testing.assert_array_equal(qp.cpu().numpy(), oracle.pool(qf_o))
    np.testing.assert_array_equal(kp.cpu().numpy(), oracle.pool(kf_o))
    # the separate entry points give the same bits
    qp2, kp2 = vsa.pool_qk(vsa.fractal_flatten(qd, shape), vsa.fractal_flatten(kd, shape), shape)
    assert torch.equal(qp, qp2) and torch.equal(kp, kp2)
    # Q and K may be the same tensor
    _, _, qp3, kp3 = vsa.flatten_pool_qk(qd, qd, shape)
    assert torch.equal(qp3, qp) and torch.equal(kp3, qp)
    vsa.device_status()


# ---------------------------------------------------------------- a3/a4 mask
def compare_csr(csr, keep_o, diag_o, thr, rows=None):
    """GPU CSR vs oracle kept flags.  Every row must match except rows whose
    boundary mass is within AMBIG_EPS of 1 - thr, which are counted.  Returns
    (#boundary rows, #mismatches there); near-tie rows are printed."""
    rp = csr.row_ptr.cpu().numpy()
    ci = csr.col_idx.cpu().numpy()
    cnt = csr.kept_count.cpu().numpy()
    nrows = rp.size - 1
    np.testing.assert_array_equal(np.diff(rp), cnt[:nrows])
    assert rp[0] == 0
    rows = np.arange(nrows) if rows is None else rows
    amb = oracle.boundary_rows(diag_o, thr, AMBIG_EPS)
    ties = oracle.near_tie_rows(diag_o, thr, AMBIG_EPS) & ~amb
    print(f"\n  {int(ties.sum())} rows with a near tie across the cut (must match)")
    Nb = keep_o.shape[1]
    bad_amb = 0
    for i, g in enumerate(rows):
        cols = ci[rp[g]:rp[g + 1]]
        assert (np.diff(cols) > 0).all() and (cols.size == 0 or (cols[0] >= 0 and cols[-1] < Nb))
        expect = np.nonzero(keep_o[i])[0]
        if amb[i]:
            bad_amb += not np.array_equal(cols, expect)
            continue
        np.testing.assert_array_equal(cols, expect, err_msg=f"row {g}")
    return int(amb.sum()), bad_amb


@pytest.mark.parametrize("name,thr,sta", [
    ("tiny", 0.2, False), ("tiny", 0.0, False), ("tiny", 0.999, True), ("tiny", 0.5, True),
    ("wan1.3b-480p", 0.2, True), ("wan1.3b-480p", 0.1, False), ("wan1.3b-480p", 0.05, True),
])
def test_block_mask_matches_oracle(name, thr, sta):
    wl = workloads.get(name)
    q, k, _ = qkv(name)
    qf, kf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k))
    qp, kp = oracle.pool(qf), oracle.pool(kf)
    keep, diag = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, thr32(thr), sta)
    csr = vsa.block_mask(dev(qp), dev(kp), vsa.Shape.of(wl), vsa.MaskParams(thr, sta))
    n_amb, bad = compare_csr(csr, keep, diag, thr32(thr))
    print(f"\n{name} thr={thr} sta={sta}: boundary rows {n_amb}/{keep.shape[0]}, differing {bad}")
    assert n_amb <= max(2, keep.shape[0] // 100)
    if thr == 0.0:
        assert int(csr.row_ptr[-1]) == keep.size
    vsa.device_status()


@pytest.mark.parametrize("T,H,W", [(2, 16, 32), (2, 96, 96)], ids=["Nb16", "Nb288"])
def test_block_mask_sta_radii_and_exact_ties(T, H, W):
    # constant Q and K: every pooled score is equal, every probability is
    # exactly 1/Nb; the CDF keeps the lowest ceil((1 - thr) * Nb) indices
    # (Nb = 288 puts more equal values at the cut than the recheck sorts)
    wl = small_shape(T=T, H=H, W=W, d=64)
    Nb = wl.Nb
    qp = np.full((1, 2, Nb, 64), 0.25)
    kp = np.full((1, 2, Nb, 64), -0.5)
    for thr, sta, radii in [(0.3, False, (1, 1, 1)), (0.7, True, (0, 1, 2)), (0.05, True, (1, 0, 0))]:
        keep, diag = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, thr32(thr), sta, radii)
        csr = vsa.block_mask(dev(qp), dev(kp), vsa.Shape.of(wl), vsa.MaskParams(thr, sta, radii))
        n_amb, bad = compare_csr(csr, keep, diag, thr32(thr))
        # every cut is an exact tie here, and the lower-index rule must decide
        # all of them identically (boundary rows included)
        assert bad == 0
        k = math.ceil((1.0 - thr32(thr)) * Nb)
        if not sta:
            assert (keep.sum(axis=1) == k).all() and keep[:, :k].all()


# ---------------------------------------------------------------- a5 attention
def attn_check(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = o_gpu.float().cpu().numpy().reshape(o_ref.shape).astype(np.float64)
    lse = lse_gpu.cpu().numpy().reshape(lse_ref.shape).astype(np.float64)
    err = np.abs(o - o_ref)
    fin = np.isfinite(lse_ref)
    lse_err = np.abs(lse[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    print(f"\n{what}: O max {err.max():.3e} mean {err.mean():.3e}; LSE max {lse_err:.3e}")
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    assert lse_err <= LSE_TOL
    assert np.array_equal(np.isneginf(lse), ~fin)


def gather_blocks(t, qblocks, Nb):
    """Rows of the listed global query blocks from a [B,h,N,...] GPU tensor."""
    flat = t.reshape(-1, 64, *t.shape[3:]) if t.dim() == 4 else t.reshape(-1, 64)
    return flat[torch.as_tensor(qblocks, device=t.device)]


@pytest.mark.parametrize("name", ["tiny", "wan1.3b-480p"])
def test_attention_with_oracle_mask(name):
    wl = workloads.get(name)
    q, k, v = qkv(name)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    keep, _ = oracle.block_mask(oracle.pool(qf), oracle.pool(kf), wl.Hb, wl.Wb,
                                thr32(wl.thr), wl.use_sta)
    rp, ci = oracle.mask_to_csr(keep)
    BH, Nb = wl.B * wl.heads, wl.Nb
    if BH * Nb <= 64:
        qb = np.arange(BH * Nb)
    else:
        rng = np.random.default_rng(5)
        cnt = np.diff(rp)
        qb = np.unique(np.concatenate([rng.choice(BH * Nb, 40, replace=False),
                                       [0, BH * Nb - 1, np.argmax(cnt), np.argmin(cnt)]]))
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci, qblocks=qb)
    o, lse = vsa.sparse_attn_fwd(dev(qf), dev(kf), dev(vf), dev(rp), dev(ci), vsa.Shape.of(wl))
    vsa.device_status()
    attn_check(gather_blocks(o, qb, Nb), gather_blocks(lse, qb, Nb), o_ref.reshape(-1, 64, wl.d),
               lse_ref.reshape(-1, 64), f"{name} oracle mask")


@pytest.mark.parametrize("T,H,W,d,density", [(3, 16, 24, 128, 0.3), (3, 16, 24, 64, 0.5),
                                             (5, 8, 16, 128, 0.05), (1, 8, 8, 64, 1.0),
                                             (2, 32, 32, 128, 0.6), (2, 32, 64, 128, 1.0),
                                             (4, 24, 40, 64, 0.15)])
def test_attention_random_mask(T, H, W, d, density):
    """Seeded random CSR (neither side's mask), with empty and single-block rows."""
    wl = small_shape(T=T, H=H, W=W, d=d)
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    BH, Nb = wl.B * wl.heads, wl.Nb
    rp, ci = workloads.random_csr(BH * Nb, Nb, density, seed=T * 1000 + H + W + d)
    # make row 1 empty and row 2 a single block (if present)
    keep = np.zeros((BH * Nb, Nb), dtype=bool)
    for g in range(BH * Nb):
        keep[g, ci[rp[g]:rp[g + 1]]] = True
    if BH * Nb > 2:
        keep[1] = False
        keep[2] = False
        keep[2, Nb - 1] = True
    HW = wl.Hb * wl.Wb
    if T >= 2 and Nb > 3:
        keep[3] = False                  # both query blocks of a time pair empty
        keep[3 + HW] = False
    rp, ci = oracle.mask_to_csr(keep)
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci)
    o, lse = vsa.sparse_attn_fwd(dev(qf), dev(kf), dev(vf), dev(rp), dev(ci), vsa.Shape.of(wl))
    vsa.device_status()
    attn_check(o, lse, o_ref.reshape(wl.B, wl.heads, wl.N, d), lse_ref.reshape(wl.B, wl.heads, wl.N),
               f"random mask {T}x{H}x{W} d={d} density={density}")


def test_attention_custom_scale_dense():
    wl = workloads.get("tiny")
    q, k, v = qkv("tiny")
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    rp, ci = oracle.mask_to_csr(np.ones((wl.heads * wl.Nb, wl.Nb), dtype=bool))
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci, scale=0.07)
    o, lse = vsa.sparse_attn_fwd(dev(qf), dev(kf), dev(vf), dev(rp), dev(ci), vsa.Shape.of(wl), 0.07)
    attn_check(o, lse, o_ref.reshape(o.shape), lse_ref.reshape(lse.shape), "dense, scale 0.07")


# ---------------------------------------------------------------- whole path
@pytest.mark.parametrize("name", ["tiny", "wan1.3b-480p"])
def test_layer_end_to_end(name):
    """flatten -> pool -> mask -> attention -> unflatten, all on the GPU, vs the
    oracle run on its own mask; attention compared on query blocks whose kept
    lists agree (all of them unless a row was reported ambiguous)."""
    wl = workloads.get(name)
    q, k, v = qkv(name)
    shape = vsa.Shape.of(wl)
    qd, kd, vd = dev(q), dev(k), dev(v)
    qf_g, kf_g, vf_g = (vsa.fractal_flatten(x, shape) for x in (qd, kd, vd))
    o_g, lse_g = vsa.attention_layer(qf_g, kf_g, vf_g, shape, vsa.MaskParams(wl.thr, wl.use_sta))
    layer = vsa.Layer(shape, vsa.MaskParams(wl.thr, wl.use_sta))
    o_g2, _ = layer(qf_g, kf_g, vf_g)
    assert torch.equal(o_g, o_g2)                        # deterministic
    o_raster = vsa.fractal_unflatten(o_g, shape)
    vsa.device_status()

    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    keep, diag = oracle.block_mask(oracle.pool(qf), oracle.pool(kf), wl.Hb, wl.Wb,
                                   thr32(wl.thr), wl.use_sta)
    rp, ci = oracle.mask_to_csr(keep)
    csr = layer.csr
    n_amb, _ = compare_csr(csr, keep, diag, thr32(wl.thr))
    BH, Nb = wl.B * wl.heads, wl.Nb
    rp_g = csr.row_ptr.cpu().numpy()
    ci_g = csr.col_idx.cpu().numpy()
    same = np.array([np.array_equal(ci_g[rp_g[g]:rp_g[g + 1]], ci[rp[g]:rp[g + 1]])
                     for g in range(BH * Nb)])
    rng = np.random.default_rng(9)
    cand = np.nonzero(same)[0]
    qb = cand if cand.size <= 64 else np.sort(rng.choice(cand, 48, replace=False))
    o_ref, lse_ref = oracle.sparse_attention(qf, kf, vf, rp, ci, qblocks=qb)
    attn_check(gather_blocks(o_g, qb, Nb), gather_blocks(lse_g, qb, Nb),
               o_ref.reshape(-1, 64, wl.d), lse_ref.reshape(-1, 64), f"{name} end to end")
    # raster-order output: row n of o_raster is flattened row f(n)
    order = oracle.fractal_order(wl.T, wl.H, wl.W)
    assert torch.equal(o_raster[0, 0, torch.as_tensor(order[:256]).cuda()], o_g[0, 0, :256])
