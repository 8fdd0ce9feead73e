"""GPU parity of the raster-layout path: pooling and block-sparse attention
that take Q, K, V in raster token order, fetch each fractal block as one
patch-shaped TMA box and store O and LSE at raster positions.

Checked bit for bit against the flattened path (flatten, pool, attention,
unflatten) on the same inputs and mask -- as is the attention that takes the
flattened tensors and stores O and LSE in raster order -- and against the oracle on sampled
query blocks: at small shapes (several tiles, odd frame counts that leave a
query tile half empty, non-square frames, d = 64 and 128, B > 1, thr = 0) and
at the full 14B 720p and 241-frame sizes in the configuration the layer
benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3

TINY = workloads.get("tiny")
SMALL = [
    TINY,                                                                  # d = 64, 4 frames
    TINY.replace(name="b2-odd-frames", B=2, T=3, H=24, W=16, d=128, use_sta=True),
    TINY.replace(name="wide-thr0", heads=3, T=5, H=16, W=40, thr=0.0),     # every block kept
    workloads.get("wan1.3b-480p"),
]


def compare(wl, n_blocks):
    shape = vsa.Shape.of(wl)
    params = vsa.MaskParams(wl.thr, wl.use_sta, wl.sta)
    q, k, v = workloads.make_qkv(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    # pooling straight from raster: the same means as the fused flatten + pool
    qf, kf, qp, kp = vsa.flatten_pool_qk(qd, kd, shape)
    qp_r, kp_r = vsa.pool_qk_raster(qd, kd, shape)
    assert torch.equal(qp_r, qp) and torch.equal(kp_r, kp)
    vf = vsa.fractal_flatten(vd, shape)
    csr = vsa.block_mask(qp, kp, shape, params)
    o_f, l_f = vsa.sparse_attn_fwd(qf, kf, vf, csr.row_ptr, csr.col_idx, shape)
    o_r, l_r = vsa.sparse_attn_fwd_raster(qd, kd, vd, csr.row_ptr, csr.col_idx, shape)
    # flattened inputs, raster outputs: the unflatten folded into the stores
    o_t, l_t = vsa.sparse_attn_fwd_to_raster(qf, kf, vf, csr.row_ptr, csr.col_idx, shape)
    vsa.device_status()
    assert torch.equal(o_t, o_r) and torch.equal(l_t, l_r)
    del qf, kf, vf, o_t, l_t
    # flattened token i sits at raster position order[i]
    order_np = oracle.fractal_order(wl.T, wl.H, wl.W)
    order = torch.as_tensor(order_np).cuda()
    assert torch.equal(o_r[:, :, order], o_f), "O differs from the flattened path"
    assert torch.equal(l_r[:, :, order], l_f), "LSE differs from the flattened path"
    del o_f, l_f
    # the layer object in raster layout runs the same calls
    layer = vsa.Layer(shape, params, qd.device, layout="raster")
    o2, l2 = layer(qd, kd, vd)
    vsa.device_status()
    assert torch.equal(o2, o_r) and torch.equal(l2, l_r)
    del layer, o2, l2
    # the oracle on sampled query blocks, on the GPU's CSR
    rp = csr.row_ptr.cpu().numpy()
    ci = csr.col_idx[:rp[-1]].cpu().numpy()
    rows = wl.B * wl.heads * wl.Nb
    rng = np.random.default_rng(17)
    pick = np.sort(rng.choice(rows, min(rows, n_blocks), replace=False))
    qf_o, kf_o, vf_o = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    o_ref, l_ref = oracle.sparse_attention(qf_o, kf_o, vf_o, rp, ci, qblocks=pick)
    bh = torch.as_tensor(pick // wl.Nb).cuda()[:, None]
    tok = torch.as_tensor(order_np[(pick % wl.Nb)[:, None] * 64 + np.arange(64)]).cuda()
    BH = wl.B * wl.heads
    og = o_r.reshape(BH, wl.N, wl.d)[bh, tok].float().cpu().numpy().reshape(o_ref.shape)
    lg = l_r.reshape(BH, wl.N)[bh, tok].cpu().numpy().reshape(l_ref.shape)
    err = np.abs(og - o_ref)
    lerr = np.abs(lg - l_ref).max()
    print(f"\n{wl.name}: {pick.size} query blocks, O max {err.max():.2e} mean {err.mean():.2e}, "
          f"LSE max {lerr:.2e}")
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    assert lerr <= LSE_TOL


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_raster_path_matches_flattened_and_oracle(wl):
    compare(wl, n_blocks=48)


@pytest.mark.parametrize("name", ["wan14b-720p", "long-241f"])
def test_raster_path_full_size(name):
    compare(workloads.get(name), n_blocks=16)
