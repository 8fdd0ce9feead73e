"""Parity at the full workload sizes, through the same calls and launch
configuration that `bench.py --layout flat` times (fused flatten+pool of Q and K, flatten of V,
block mask, sparse attention, unflatten of O, all heads in one launch each).

The oracle cannot run a whole 40-head or 24-head layer in a test, so it checks
sampled outputs one by one: a few heads in full for flatten and pool (bit
exact), sampled mask rows (bit exact except rows whose boundary mass lies
within 1e-5 of 1 - thr, which are reported), and sampled query blocks of attention (O and LSE
within tolerance, on the GPU's own CSR).  Properties that hold at any size are
checked over the whole output: CSR structure, non-empty rows, STA window
coverage, finite O and LSE, and the unflatten permutation on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3
AMBIG_EPS = 1e-5


def thr32(thr):
    return float(np.float32(thr))


def u16(t):
    return oracle.as_u16(t.cpu())


def run_path(wl):
    """The bench's step on the whole workload; returns every intermediate."""
    shape = vsa.Shape.of(wl)
    params = vsa.MaskParams(wl.thr, wl.use_sta, wl.sta)
    q, k, v = workloads.make_qkv(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    layer = vsa.Layer(shape, params, qd.device)
    qf, kf = torch.empty_like(qd), torch.empty_like(kd)
    vsa.flatten_pool_qk(qd, kd, shape, out=(qf, kf, layer.qp, layer.kp))
    vf = vsa.fractal_flatten(vd, shape)
    vsa.block_mask(layer.qp, layer.kp, shape, params, out=layer.csr, workspace=layer.ws_mask)
    vsa.sparse_attn_fwd(qf, kf, vf, layer.csr.row_ptr, layer.csr.col_idx, shape, 0.0,
                        out=(layer.o, layer.lse), workspace=layer.ws_attn)
    o_raster = vsa.fractal_unflatten(layer.o, shape)
    vsa.device_status()
    return (q, k, v), (qf, kf, vf), layer, o_raster


def check_csr_properties(wl, csr):
    """Whole-output invariants of the block mask."""
    Nb, rows = wl.Nb, wl.B * wl.heads * wl.Nb
    rp = csr.row_ptr
    cnt = csr.kept_count[:rows].to(torch.int64)
    assert int(rp[0]) == 0
    assert torch.equal(rp[1:] - rp[:-1], cnt)
    assert int(cnt.min()) >= 1, "a row kept no block (its argmax block is always kept)"
    nnz = int(rp[-1])
    ci = csr.col_idx[:nnz].to(torch.int64)
    assert int(ci.min()) >= 0 and int(ci.max()) < Nb
    row_of = torch.repeat_interleave(torch.arange(rows, device=ci.device), cnt)
    same_row = row_of[1:] == row_of[:-1]
    assert bool((ci[1:][same_row] > ci[:-1][same_row]).all()), "columns not strictly ascending"
    if wl.use_sta:
        # every kept list contains the row's clipped Chebyshev window
        HW = wl.Hb * wl.Wb
        r = row_of % Nb
        rt, ry, rx = r // HW, (r % HW) // wl.Wb, r % wl.Wb
        ct, cy, cx = ci // HW, (ci % HW) // wl.Wb, ci % wl.Wb
        st, sh, sw = wl.sta
        inside = ((ct - rt).abs() <= st) & ((cy - ry).abs() <= sh) & ((cx - rx).abs() <= sw)
        in_win = torch.zeros(rows, dtype=torch.int64, device=ci.device)
        in_win.index_add_(0, row_of, inside.to(torch.int64))
        g = torch.arange(rows, device=ci.device) % Nb
        gt, gy, gx = g // HW, (g % HW) // wl.Wb, g % wl.Wb

        def span(c, rad, n):
            return torch.clamp(c + rad, max=n - 1) - torch.clamp(c - rad, min=0) + 1
        want = span(gt, st, wl.T) * span(gy, sh, wl.Hb) * span(gx, sw, wl.Wb)
        assert torch.equal(in_win, want), "an STA window block is missing"
    return nnz


def sample_rows(wl, counts_head, rng, n_random=20):
    """Query-block rows of one head to check: random ones, the grid's corner
    and frame-edge rows, and the rows with the most and fewest kept blocks."""
    Nb, HW = wl.Nb, wl.Hb * wl.Wb
    fixed = {0, Nb - 1, HW - 1, (wl.T - 1) * HW, (wl.T // 2) * HW + HW // 2,
             int(np.argmax(counts_head)), int(np.argmin(counts_head))}
    rnd = set(rng.choice(Nb, n_random, replace=False).tolist())
    return np.array(sorted(fixed | rnd), dtype=np.int64)


@pytest.mark.parametrize("name", ["wan14b-720p", "long-241f"])
def test_full_size_sampled(name):
    wl = workloads.get(name)
    (q, k, v), (qf, kf, vf), layer, o_raster = run_path(wl)
    csr = layer.csr
    Nb = wl.Nb
    nnz = check_csr_properties(wl, csr)
    assert bool(torch.isfinite(layer.lse).all()), "non-finite LSE"
    assert bool(torch.isfinite(layer.o.float()).all()), "non-finite O"
    rng = np.random.default_rng(2718)
    heads = sorted({0, wl.heads // 2, wl.heads - 1})
    rp_g = csr.row_ptr.cpu().numpy()
    ci_g = csr.col_idx[:nnz].cpu().numpy()
    cnt_g = csr.kept_count.cpu().numpy()
    thr = thr32(wl.thr)
    n_amb = n_bad_amb = n_tie = 0
    for h in heads:
        # flatten and pool of this head: bit exact
        qf_o, kf_o, vf_o = (oracle.flatten(x[:, h:h + 1], wl.T, wl.H, wl.W) for x in (q, k, v))
        np.testing.assert_array_equal(u16(qf[:, h:h + 1]), qf_o)
        np.testing.assert_array_equal(u16(kf[:, h:h + 1]), kf_o)
        np.testing.assert_array_equal(u16(vf[:, h:h + 1]), vf_o)
        qp_o, kp_o = oracle.pool(qf_o), oracle.pool(kf_o)
        np.testing.assert_array_equal(layer.qp[:, h:h + 1].cpu().numpy(), qp_o)
        np.testing.assert_array_equal(layer.kp[:, h:h + 1].cpu().numpy(), kp_o)
        # mask rows: bit exact except rows reported within rounding of the cut
        base = h * Nb                                   # B = 1 in every full-size workload
        rows = sample_rows(wl, cnt_g[base:base + Nb], rng)
        keep, diag = oracle.block_mask(qp_o, kp_o, wl.Hb, wl.Wb, thr, wl.use_sta, wl.sta,
                                       rows=rows)
        amb = oracle.boundary_rows(diag, thr, AMBIG_EPS)
        n_tie += int((oracle.near_tie_rows(diag, thr, AMBIG_EPS) & ~amb).sum())
        for i, r in enumerate(rows):
            g = base + r
            got = ci_g[rp_g[g]:rp_g[g + 1]]
            want = np.nonzero(keep[i])[0]
            if amb[i]:
                n_amb += 1
                n_bad_amb += not np.array_equal(got, want)
                continue
            np.testing.assert_array_equal(got, want, err_msg=f"{name} head {h} row {r}")
        # attention on the GPU's CSR for those query blocks
        sub_rp = (rp_g[base:base + Nb + 1] - rp_g[base]).astype(np.int64)
        sub_ci = ci_g[rp_g[base]:rp_g[base + Nb]]
        o_ref, lse_ref = oracle.sparse_attention(qf_o, kf_o, vf_o, sub_rp, sub_ci, qblocks=rows)
        o_g = layer.o[0, h].reshape(Nb, 64, wl.d)[torch.as_tensor(rows).cuda()]
        l_g = layer.lse[0, h].reshape(Nb, 64)[torch.as_tensor(rows).cuda()]
        o = o_g.float().cpu().numpy().reshape(o_ref.shape).astype(np.float64)
        lse = l_g.cpu().numpy().reshape(lse_ref.shape).astype(np.float64)
        err = np.abs(o - o_ref)
        lse_err = np.abs(lse - lse_ref).max()
        print(f"\n{name} head {h}: {rows.size} query blocks, O max {err.max():.3e} "
              f"mean {err.mean():.3e}; LSE max {lse_err:.3e}")
        assert err.max() <= O_MAX and err.mean() <= O_MEAN
        assert lse_err <= LSE_TOL
        # unflatten: flattened token i sits at raster position order[i]
        order = oracle.fractal_order(wl.T, wl.H, wl.W)
        tok = np.sort(rng.choice(wl.N, 4096, replace=False))
        assert torch.equal(o_raster[0, h, torch.as_tensor(order[tok]).cuda()],
                           layer.o[0, h, torch.as_tensor(tok).cuda()])
    print(f"{name}: nnz {nnz} ({nnz / (wl.heads * Nb * Nb):.4f} kept), "
          f"{n_amb} sampled rows with the boundary mass within {AMBIG_EPS} of 1 - thr, "
          f"{n_bad_amb} of them differ; {n_tie} near-tie rows matched")
