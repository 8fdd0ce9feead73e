"""Attention item structures that stress the kernel's hand-offs between
consecutive work items, compared with the oracle on sampled query blocks.

A work item is a 128-row tile (two query blocks of one head) that walks the
merged kept lists two key blocks per step.  When every item has a single step,
each item's last step directly follows the previous item's last step, taken
by the other softmax group: the case in which the epilogue's wait for a
complete O must name its own item and not the one before it.  The STA window
of radius 0 (each block keeps only itself) and random lists of one or two
blocks per row produce exactly such items, at the Wan-14B 720p grid.

The planner sorts each head's items longest first with a single-CTA sort of
at most 4096 items per head; larger heads take the items in index order
instead.  A 2 x 512 x 576 grid (4608 time-paired items per head) reaches that
branch.
"""
import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


def _check_sampled(wl, q, k, v, o, lse, rp, ci, heads, rng, n_blocks=48, what=""):
    """Oracle attention on sampled query blocks of the given heads."""
    Nb = wl.Nb
    for j, h in enumerate(heads):
        qf_o, kf_o, vf_o = (oracle.flatten(x[:, j:j + 1], wl.T, wl.H, wl.W) for x in (q, k, v))
        base = h * Nb
        sub_rp = (rp[base:base + Nb + 1] - rp[base]).astype(np.int64)
        sub_ci = ci[rp[base]:rp[base + Nb]]
        rows = np.unique(np.concatenate([[0, 1, Nb - 1],
                                         rng.choice(Nb, n_blocks, replace=False)]))
        o_ref, lse_ref = oracle.sparse_attention(qf_o, kf_o, vf_o, sub_rp, sub_ci, qblocks=rows)
        idx = torch.as_tensor(rows).cuda()
        o_g = o[0, h].reshape(Nb, 64, wl.d)[idx].float().cpu().numpy().astype(np.float64)
        l_g = lse[0, h].reshape(Nb, 64)[idx].cpu().numpy().astype(np.float64)
        err = np.abs(o_g.reshape(o_ref.shape) - o_ref)
        lse_err = np.abs(l_g.reshape(lse_ref.shape) - lse_ref).max()
        print(f"\n{what} head {h}: {rows.size} blocks, O max {err.max():.3e} "
              f"mean {err.mean():.3e}; LSE max {lse_err:.3e}")
        assert err.max() <= O_MAX and err.mean() <= O_MEAN
        assert lse_err <= LSE_TOL


def _flat_inputs(wl, heads):
    q, k, v = workloads.make_qkv(wl, heads=heads)
    shape = vsa.Shape(wl.B, len(heads), wl.T, wl.H, wl.W, wl.d)
    qf, kf, vf = (vsa.fractal_flatten(x.cuda(), shape) for x in (q, k, v))
    return (q, k, v), shape, (qf, kf, vf)


@pytest.mark.parametrize("mask", ["sta-radius-0", "one-or-two-blocks"])
def test_single_step_items_back_to_back(mask):
    wl = workloads.get("wan14b-720p").replace(name="wan14b-720p-items", heads=8)
    heads = list(range(wl.heads))
    (q, k, v), shape, (qf, kf, vf) = _flat_inputs(wl, heads)
    rows = wl.B * len(heads) * wl.Nb
    if mask == "sta-radius-0":
        csr = vsa.sta_mask(shape, radii=(0, 0, 0))
        rp_d, ci_d = csr.row_ptr, csr.col_idx
        rp = rp_d.cpu().numpy()
        ci = ci_d[:int(rp[-1])].cpu().numpy()
        # every row keeps exactly its own block: one step per item
        assert np.array_equal(np.diff(rp), np.ones(rows, dtype=np.int64))
        assert np.array_equal(ci, np.tile(np.arange(wl.Nb, dtype=np.int32), len(heads)))
    else:
        rp, ci = workloads.short_csr(rows, wl.Nb, 1, 2, seed=4242)
        rp_d, ci_d = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    o, lse = vsa.sparse_attn_fwd(qf, kf, vf, rp_d, ci_d, shape)
    # the same launch again: the scheduler's counter and plan are rebuilt
    o2, lse2 = vsa.sparse_attn_fwd(qf, kf, vf, rp_d, ci_d, shape)
    vsa.device_status()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert bool(torch.isfinite(lse).all())
    rng = np.random.default_rng(31)
    sample = sorted({0, 3, wl.heads - 1})
    sel = [heads.index(h) for h in sample]
    _check_sampled(wl, q[:, sel], k[:, sel], v[:, sel], o, lse, rp, ci, sample, rng,
                   what=f"14B grid, {mask}")


def test_heads_beyond_the_sorting_planner():
    """More than 4096 items per head: items run in index order (no per-head
    sort); the result must not depend on the order."""
    wl = workloads.Workload("wide", B=1, heads=2, d=64, T=2, H=512, W=576, clusters=4,
                            thr=0.2, use_sta=False, seed=91)
    assert ((wl.T + 1) // 2) * wl.Hb * wl.Wb > 4096
    heads = [0, 1]
    (q, k, v), shape, (qf, kf, vf) = _flat_inputs(wl, heads)
    rows = len(heads) * wl.Nb
    rp, ci = workloads.short_csr(rows, wl.Nb, 1, 6, seed=777)
    o, lse = vsa.sparse_attn_fwd(qf, kf, vf, torch.from_numpy(rp).cuda(),
                                 torch.from_numpy(ci).cuda(), shape)
    vsa.device_status()
    assert bool(torch.isfinite(lse).all())
    _check_sampled(wl, q, k, v, o, lse, rp, ci, heads, np.random.default_rng(5),
                   what="4608 items per head")
