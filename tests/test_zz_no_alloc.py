"""vsa_sparse_attn_fwd_noalloc: the attention entry point for callers that
cannot allocate device memory (plugins handed only inputs and outputs,
processes that reserve all device memory up front, latency-critical paths
where cudaMalloc would synchronise the device).  Called through the C ABI and
checked against vsa_sparse_attn_fwd, which takes a caller workspace, on two
calls in a row (the shared built-in scratch must be re-planned each time)."""
import ctypes

import numpy as np
import pytest
import torch

from content_adaptive_block_fractal_b200 import _lib, workloads
import content_adaptive_block_fractal_b200 as vsa


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(wl, density, seed):
    q, k, v = workloads.make_qkv(wl)
    shape = vsa.Shape.of(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    qf, kf, vf = (vsa.fractal_flatten(x, shape) for x in (qd, kd, vd))
    rp, ci = workloads.random_csr(wl.B * wl.heads * wl.Nb, wl.Nb, density, seed)
    return shape, qf, kf, vf, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()


def _with_workspace(L, shape, qf, kf, vf, rp, ci, stream):
    o = torch.empty_like(qf)
    lse = torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=qf.device)
    ws = torch.empty(vsa.sparse_attn_workspace_size(shape), dtype=torch.uint8, device=qf.device)
    _lib.check(L.vsa_sparse_attn_fwd(_p(qf), _p(kf), _p(vf), _p(rp), _p(ci), shape.c(), 0.0,
                                     _p(o), _p(lse), _p(ws), ws.numel(), stream))
    return o, lse


def _no_alloc(L, shape, qf, kf, vf, rp, ci, stream):
    o = torch.empty_like(qf)
    lse = torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=qf.device)
    _lib.check(L.vsa_sparse_attn_fwd_noalloc(_p(qf), _p(kf), _p(vf), _p(rp), _p(ci), shape.c(),
                                             0.0, _p(o), _p(lse), stream))
    return o, lse


def _same(a, b):
    """Both entry points run the same kernel on the same inputs, and each
    128-row tile is computed by one CTA in a fixed order, so O and LSE must
    agree bit for bit (a stale plan or an aliased scratch would not)."""
    (oa, la), (ob, lb) = a, b
    assert torch.equal(oa, ob)
    assert torch.equal(la, lb)


@pytest.mark.gpu
def test_no_alloc_matches_workspace_entry_point_twice():
    L = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        (workloads.Workload("grid-a", B=1, heads=3, d=128, T=5, H=32, W=32, clusters=4, thr=0.2,
                            use_sta=False, seed=41, seeds_3d=True), 0.2, 1),
        (workloads.Workload("grid-b", B=2, heads=2, d=64, T=4, H=16, W=24, clusters=4, thr=0.2,
                            use_sta=False, seed=42, seeds_3d=True), 0.4, 2),
    ]
    for wl, density, seed in cases:
        shape, qf, kf, vf, rp, ci = _inputs(wl, density, seed)
        ref = _with_workspace(L, shape, qf, kf, vf, rp, ci, stream)
        first = _no_alloc(L, shape, qf, kf, vf, rp, ci, stream)
        second = _no_alloc(L, shape, qf, kf, vf, rp, ci, stream)
        torch.cuda.synchronize()
        _lib.check(L.vsa_device_status(stream))
        _same(first, ref)
        _same(second, ref)


@pytest.mark.gpu
def test_no_alloc_rejects_shapes_beyond_its_scratch():
    L = _lib.load()
    big = vsa.Shape(1, 2100, 2, 256, 256, 128)          # ~2.15M query tiles: > 8 MiB of scratch
    assert vsa.sparse_attn_workspace_size(big) > (8 << 20)
    P = ctypes.c_void_p
    st = L.vsa_sparse_attn_fwd_noalloc(P(1 << 12), P(1 << 16), P(1 << 20), P(1 << 24),
                                       P(1 << 26), big.c(), 0.0, P(1 << 28), P(1 << 29), None)
    assert st == 3
    assert b"scratch" in L.vsa_last_error()
