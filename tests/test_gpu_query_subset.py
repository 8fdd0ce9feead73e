"""GPU parity of query-subset attention (only listed query blocks are
computed; the rest of O and LSE is left untouched) against the oracle."""
import functools

import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import workloads

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


@functools.lru_cache(maxsize=2)
def setup(name, thr):
    wl = workloads.get(name)
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    rows = wl.B * wl.heads * wl.Nb
    if thr is None:        # every block kept: HSA's full-context attention
        keep = np.ones((rows, wl.Nb), dtype=np.uint8)
    else:
        keep, _ = oracle.block_mask(oracle.pool(qf), oracle.pool(kf), wl.Hb, wl.Wb,
                                    float(np.float32(thr)), wl.use_sta)
    rp, ci = oracle.mask_to_csr(keep)
    return wl, (qf, kf, vf), (rp, ci)


def dev(x):
    if x.dtype == np.uint16:
        return oracle.to_bf16_tensor(x).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def subsets(wl, rng):
    rows = wl.B * wl.heads * wl.Nb
    HW = wl.Hb * wl.Wb
    r = np.arange(rows)
    frame = (r % wl.Nb) // HW
    return {
        "random30": np.sort(rng.choice(rows, max(1, rows * 3 // 10), replace=False)),
        "odd_frames": r[frame % 2 == 1],               # no block has its partner listed
        "even_frames": r[frame % 2 == 0],
        "one": np.array([rows // 2 + 1]),
        "all": r,
    }


@pytest.mark.parametrize("name,thr", [("tiny", 0.2), ("wan1.3b-480p", 0.2),
                                      ("wan1.3b-480p", None)])
def test_query_subset_matches_oracle(name, thr):
    wl, (qf, kf, vf), (rp, ci) = setup(name, thr)
    shape = vsa.Shape.of(wl)
    qd, kd, vd = dev(qf), dev(kf), dev(vf)
    rpd, cid = dev(rp), dev(ci.astype(np.int32))
    rng = np.random.default_rng(11)
    o_full, l_full = vsa.sparse_attn_fwd(qd, kd, vd, rpd, cid, shape)
    for label, qb in subsets(wl, rng).items():
        o = torch.full_like(qd, 7.0)
        lse = torch.full((shape.B, shape.heads, shape.N), 123.0, device="cuda")
        vsa.sparse_attn_fwd_rows(qd, kd, vd, rpd, cid, shape, torch.as_tensor(qb), out=(o, lse))
        vsa.device_status()
        listed = np.zeros(wl.B * wl.heads * wl.Nb, dtype=bool)
        listed[qb] = True
        ob = o.reshape(-1, 64, wl.d)
        lb = lse.reshape(-1, 64)
        untouched = torch.as_tensor(np.nonzero(~listed)[0]).cuda()
        assert bool((ob[untouched] == 7.0).all()) and bool((lb[untouched] == 123.0).all()), label
        # computed blocks: the oracle on a sample of them
        pick = qb if qb.size <= 48 else np.sort(rng.choice(qb, 48, replace=False))
        o_ref, l_ref = oracle.sparse_attention(qf, kf, vf, rp, ci, qblocks=pick)
        og = ob[torch.as_tensor(pick).cuda()].float().cpu().numpy().reshape(o_ref.shape)
        lg = lb[torch.as_tensor(pick).cuda()].cpu().numpy().reshape(-1)
        err = np.abs(og - o_ref)
        print(f"\n{name} thr={thr} {label}: {qb.size} blocks, O max {err.max():.2e} "
              f"mean {err.mean():.2e}, LSE max {np.abs(lg - l_ref).max():.2e}")
        assert err.max() <= O_MAX and err.mean() <= O_MEAN, label
        assert np.abs(lg - l_ref).max() <= LSE_TOL, label
        if label == "all":
            # every block listed: the same values as the full call
            d = (o.float() - o_full.float()).abs().max().item()
            assert d <= 2e-2 and (lse - l_full).abs().max().item() <= LSE_TOL


def test_query_subset_unsorted_list_is_reported():
    wl, (qf, kf, vf), (rp, ci) = setup("tiny", 0.2)
    shape = vsa.Shape.of(wl)
    qb = torch.tensor([5, 3, 9], dtype=torch.int32)      # 3 is out of order: skipped
    o = torch.zeros_like(dev(qf))
    lse = torch.zeros((shape.B, shape.heads, shape.N), device="cuda")
    vsa.sparse_attn_fwd_rows(dev(qf), dev(kf), dev(vf), dev(rp), dev(ci.astype(np.int32)),
                             shape, qb, out=(o, lse))
    with pytest.raises(vsa.VsaError, match="bad block index"):
        vsa.device_status()
    vsa.device_status()                                   # the word was cleared
    lb = lse.reshape(-1, 64)
    assert bool((lb[5] != 0).all())                       # a valid lead is computed
    assert bool(torch.isfinite(lb).all())
