"""Pins for the CPU oracle, against things other than the oracle itself.

Each check ties one oracle function to a hand-derived fixture, a closed form,
brute force, or a library routine the oracle does not use (numpy mean, torch
softmax, torch scaled_dot_product_attention), chosen so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from content_adaptive_block_fractal_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- O1 flatten
def test_fractal_order_matches_hand_derived_golden():
    expect = np.array([int(x) for x in _lines("fractal_order_T2_H4_W4_P2.txt")])
    np.testing.assert_array_equal(oracle.fractal_order(2, 4, 4, 2), expect)


@pytest.mark.parametrize("T,H,W,P", [(3, 16, 24, 8), (1, 8, 8, 8), (2, 6, 4, 2), (4, 16, 16, 8)])
def test_fractal_order_is_patch_contiguous_bijection(T, H, W, P):
    order = oracle.fractal_order(T, H, W, P)
    N = T * H * W
    assert sorted(order.tolist()) == list(range(N))            # bijection
    t, rem = np.divmod(order, H * W)
    y, x = np.divmod(rem, W)
    blk = P * P
    # every run of P*P flattened tokens is one patch of one frame ...
    for b in range(N // blk):
        sl = slice(b * blk, (b + 1) * blk)
        assert len(set(t[sl])) == 1 and len(set(y[sl] // P)) == 1 and len(set(x[sl] // P)) == 1
        # ... listed row-major inside the patch
        np.testing.assert_array_equal((y[sl] % P) * P + x[sl] % P, np.arange(blk))
    # patches follow (frame, patch row, patch col) in lexicographic order
    key = (t[::blk] * (H // P) + y[::blk] // P) * (W // P) + x[::blk] // P
    np.testing.assert_array_equal(key, np.arange(N // blk))


def test_fractal_order_identity_when_patch_covers_frame():
    np.testing.assert_array_equal(oracle.fractal_order(5, 8, 8, 8), np.arange(5 * 64))


def test_flatten_unflatten_roundtrip():
    wl = workloads.get("tiny")
    q, _, _ = workloads.make_qkv(wl)
    qf = oracle.flatten(q, wl.T, wl.H, wl.W)
    back = oracle.unflatten(qf, wl.T, wl.H, wl.W)
    np.testing.assert_array_equal(back, oracle.as_u16(q))
    # the gather really moved rows: row k of qf is raster row order[k]
    order = oracle.fractal_order(wl.T, wl.H, wl.W)
    np.testing.assert_array_equal(qf[0, 1, 77], oracle.as_u16(q)[0, 1, order[77]])


# ---------------------------------------------------------------- O2 pool
def test_pool_equals_numpy_block_mean():
    wl = workloads.get("tiny")
    q, _, _ = workloads.make_qkv(wl)
    qp = oracle.pool(q)
    ref = q.double().numpy().reshape(wl.B, wl.heads, wl.Nb, 64, wl.d).mean(axis=3)
    # randn data spans far less than 2^39 per block, so every sum of 64 bf16
    # values is exact in fp64 and the mean is exact in any summation order
    np.testing.assert_array_equal(qp, ref)


def test_pool_constant_block_and_linearity():
    x = torch.zeros(1, 128, 8, dtype=torch.bfloat16)
    x[0, :64] = 1.5
    x[0, 64:] = torch.arange(64, dtype=torch.float32)[:, None]   # 0..63
    p = oracle.pool(x)
    np.testing.assert_array_equal(p[0, 0], np.full(8, 1.5))
    np.testing.assert_array_equal(p[0, 1], np.full(8, 31.5))      # closed form (0+63)/2


# ---------------------------------------------------------------- O3 reduced attention
def test_reduced_attention_matches_torch_softmax():
    rng = np.random.default_rng(5)
    qp = rng.standard_normal((3, 20, 16))
    kp = rng.standard_normal((3, 20, 16))
    a = oracle.reduced_attention(qp, kp).reshape(3, 20, 20)
    ref = torch.softmax(torch.from_numpy(qp) @ torch.from_numpy(kp).transpose(1, 2) / 4.0, dim=-1)
    np.testing.assert_allclose(a, ref.numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(a.sum(axis=-1), 1.0, rtol=1e-14)


def test_reduced_attention_two_blocks_closed_form():
    qp = np.array([[[1.0, 2.0], [0.5, -1.0]]])
    kp = np.array([[[3.0, -1.0], [0.0, 2.0]]])
    a = oracle.reduced_attention(qp, kp)
    s = qp[0] @ kp[0].T / math.sqrt(2.0)
    for r in range(2):
        p0 = 1.0 / (1.0 + math.exp(s[r, 1] - s[r, 0]))        # two-way softmax = logistic
        assert a[r, 0] == pytest.approx(p0, rel=1e-14)
        assert a[r, 1] == pytest.approx(1.0 - p0, rel=1e-13)


def test_reduced_attention_row_subset():
    rng = np.random.default_rng(6)
    qp = rng.standard_normal((2, 9, 8))
    kp = rng.standard_normal((2, 9, 8))
    full = oracle.reduced_attention(qp, kp)
    rows = np.array([0, 10, 17])
    np.testing.assert_array_equal(oracle.reduced_attention(qp, kp, rows), full[rows])


# ---------------------------------------------------------------- O4 selection
def test_select_matches_hand_worked_rows():
    for ln in _lines("topp_rows.txt"):
        thr, p, kept = (part.strip() for part in ln.split("|"))
        keep, _ = oracle.select_row(np.array([float(x) for x in p.split()]), float(thr))
        assert np.nonzero(keep)[0].tolist() == [int(x) for x in kept.split()], ln


def _brute_force(w, target):
    """Minimum-cardinality subset with mass >= target; among those the one of
    largest mass, then the lexicographically smallest index list."""
    n = len(w)
    for size in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), size):
            m = sum(w[i] for i in sub)
            if m >= target and (best is None or m > best[0] or (m == best[0] and sub < best[1])):
                best = (m, sub)
        if best is not None:
            return set(best[1])
    return set(range(n))


@pytest.mark.parametrize("seed", range(60))
def test_select_equals_brute_force_on_small_rows(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 13))
    # small integer weights (many ties), completed so that they sum to 2^k:
    # every probability and every partial sum is then an exact dyadic
    w = rng.integers(0, 8, size=n - 1).tolist()
    k = max(1, int(sum(w)).bit_length())
    w.append((1 << k) - sum(w))
    rng.shuffle(w)
    total = 1 << k
    p = np.array(w, dtype=np.float64) / total
    thr_num = int(rng.integers(0, total))
    thr = thr_num / total
    keep, diag = oracle.select_row(p, thr)
    if thr == 0.0:
        assert keep.all()
        return
    expect = _brute_force(w, total - thr_num)
    assert set(np.nonzero(keep)[0].tolist()) == expect, (w, thr_num)
    assert diag[4] == len(expect)


@pytest.mark.parametrize("thr", [0.0, 0.05, 0.1, 0.3, 0.9])
def test_select_minimality_invariant(thr):
    rng = np.random.default_rng(7)
    for _ in range(50):
        a = rng.dirichlet(np.full(300, 0.2))
        keep, diag = oracle.select_row(a, thr)
        kept = np.sort(a[keep])[::-1]
        if thr == 0.0:
            assert keep.all()
            continue
        assert kept.sum() >= 1.0 - thr - 1e-12              # enough mass
        assert kept[:-1].sum() < 1.0 - thr                   # no proper prefix suffices
        dropped = a[~keep]
        assert dropped.size == 0 or dropped.max() <= kept.min()   # kept = a top set
        assert diag[0] == pytest.approx(kept.sum(), rel=1e-12)


def test_sta_window_matches_hand_derived_golden():
    for ln in _lines("sta_window_T3_Hb3_Wb3_r1.txt"):
        r, cols = ln.split(":")
        got = [c for c in range(27) if oracle.sta_keep(int(r), c, 3, 3)]
        assert got == [int(c) for c in cols.split()]


def test_sta_window_counts_closed_form():
    T, Hb, Wb = 4, 5, 6
    for rt, rh, rw in [(1, 1, 1), (0, 2, 1), (2, 0, 0)]:
        for r in range(T * Hb * Wb):
            t, py, px = r // (Hb * Wb), (r // Wb) % Hb, r % Wb
            width = lambda c, rad, n: min(c + rad, n - 1) - max(c - rad, 0) + 1
            expect = width(t, rt, T) * width(py, rh, Hb) * width(px, rw, Wb)
            got = sum(oracle.sta_keep(r, c, Hb, Wb, rt, rh, rw) for c in range(T * Hb * Wb))
            assert got == expect


def test_block_mask_union_and_threshold_extremes():
    wl = workloads.get("tiny")
    q, k, _ = workloads.make_qkv(wl)
    qf = oracle.flatten(q, wl.T, wl.H, wl.W)
    kf = oracle.flatten(k, wl.T, wl.H, wl.W)
    qp, kp = oracle.pool(qf), oracle.pool(kf)
    keep0, _ = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, 0.0, False)
    assert keep0.all()                                          # thr = 0 keeps everything
    a = oracle.reduced_attention(qp, kp)
    for thr in (0.2, 0.6):
        knab, diag = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, thr, False)
        kuni, _ = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, thr, True)
        assert (kuni >= knab).all()                             # union contains NABLA part
        for row in range(a.shape[0]):
            r = row % wl.Nb
            sta = [oracle.sta_keep(r, c, wl.Hb, wl.Wb) for c in range(wl.Nb)]
            assert all(kuni[row, c] for c in range(wl.Nb) if sta[c])
            assert (knab[row] == oracle.select_row(a[row], thr)[0]).all()
            assert knab[row, np.argmax(a[row])]                # argmax always kept
    # thr close to 1 keeps only the argmax, so the STA part dominates
    kmax, _ = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, 1.0 - 1e-9, False)
    assert (kmax.sum(axis=1) == 1).all()


# ---------------------------------------------------------------- O5 attention
def _sdpa_f64(q, k, v, mask=None):
    q, k, v = (torch.as_tensor(x, dtype=torch.float64) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)


def test_attention_all_blocks_equals_dense_sdpa():
    wl = workloads.get("tiny")
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    BH, Nb = wl.B * wl.heads, wl.Nb
    rp, ci = oracle.mask_to_csr(np.ones((BH * Nb, Nb), dtype=bool))
    o, lse = oracle.sparse_attention(qf, kf, vf, rp, ci)
    ref = _sdpa_f64(*(oracle.to_bf16_tensor(x).double() for x in (qf, kf, vf)))
    np.testing.assert_allclose(o.reshape(ref.shape), ref.numpy(), rtol=0, atol=1e-12)
    s = torch.from_numpy(oracle.to_bf16_tensor(qf).double().numpy()) @ \
        torch.from_numpy(oracle.to_bf16_tensor(kf).double().numpy()).transpose(-1, -2) / math.sqrt(wl.d)
    np.testing.assert_allclose(lse.reshape(s.shape[:-1]), torch.logsumexp(s, -1).numpy(), rtol=1e-13)


def test_attention_permutation_equivariance_against_raster_dense():
    """unflatten(attn(flatten(q, k, v))) equals dense attention in raster order."""
    wl = workloads.get("tiny")
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    BH, Nb = wl.B * wl.heads, wl.Nb
    rp, ci = oracle.mask_to_csr(np.ones((BH * Nb, Nb), dtype=bool))
    o, _ = oracle.sparse_attention(qf, kf, vf, rp, ci)
    o_raster = oracle.unflatten_f64(o.reshape(wl.B, wl.heads, wl.N, wl.d), wl.T, wl.H, wl.W)
    ref = _sdpa_f64(q.double(), k.double(), v.double())
    np.testing.assert_allclose(o_raster, ref.numpy(), rtol=0, atol=1e-12)


def test_attention_random_block_mask_equals_masked_sdpa():
    wl = workloads.get("tiny")
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    BH, Nb = wl.B * wl.heads, wl.Nb
    rp, ci = workloads.random_csr(BH * Nb, Nb, 0.3, seed=11)
    o, lse = oracle.sparse_attention(qf, kf, vf, rp, ci)
    keep = np.zeros((BH * Nb, Nb), dtype=bool)
    for g in range(BH * Nb):
        keep[g, ci[rp[g]:rp[g + 1]]] = True
    tok = np.repeat(np.repeat(keep.reshape(BH, Nb, Nb), 64, axis=1), 64, axis=2)
    mask = torch.from_numpy(tok).reshape(wl.B, wl.heads, wl.N, wl.N)
    Q, K, V = (oracle.to_bf16_tensor(x).double() for x in (qf, kf, vf))
    ref = _sdpa_f64(Q, K, V, mask)
    np.testing.assert_allclose(o.reshape(ref.shape), ref.numpy(), rtol=0, atol=1e-12)
    s = (Q @ K.transpose(-1, -2) / math.sqrt(wl.d)).masked_fill(~mask, -math.inf)
    np.testing.assert_allclose(lse.reshape(s.shape[:-1]), torch.logsumexp(s, -1).numpy(), rtol=1e-13)


def test_attention_single_block_rows_and_empty_rows():
    rng = np.random.default_rng(3)
    N, d = 256, 32
    qf = torch.from_numpy(rng.standard_normal((1, N, d))).to(torch.bfloat16)
    kf = torch.from_numpy(rng.standard_normal((1, N, d))).to(torch.bfloat16)
    vf = torch.from_numpy(rng.standard_normal((1, N, d))).to(torch.bfloat16)
    rp = np.array([0, 1, 2, 2, 3], dtype=np.int64)          # block 2 has no keys
    ci = np.array([3, 0, 1], dtype=np.int32)
    o, lse = oracle.sparse_attention(qf, kf, vf, rp, ci, scale=0.25)
    Q, K, V = qf.double()[0], kf.double()[0], vf.double()[0]
    for qb, kb in [(0, 3), (1, 0), (3, 1)]:
        qs, ks = slice(qb * 64, qb * 64 + 64), slice(kb * 64, kb * 64 + 64)
        ref = torch.softmax(Q[qs] @ K[ks].T * 0.25, -1) @ V[ks]
        np.testing.assert_allclose(o[qs], ref.numpy(), atol=1e-12)
    np.testing.assert_array_equal(o[128:192], 0.0)
    assert np.isneginf(lse[128:192]).all()


def test_ambiguity_classifier():
    diag = np.array([[0.92, 0.85, 0.07, 0.01, 3],     # clear
                     [0.900004, 0.8, 0.1, 0.01, 2],    # kept mass within 1e-5 of 0.9
                     [0.95, 0.899995, 0.05, 0.01, 4],  # mass without last block within 1e-5
                     [0.95, 0.85, 0.1, 0.0999995, 5],  # near tie across the cut
                     [1.0, 0.85, 0.15, -1.0, 9]])      # nothing dropped
    np.testing.assert_array_equal(oracle.ambiguous_rows(diag, 0.1),
                                  [False, True, True, True, False])


# ---------------------------------------------------------------- f2 static ratio (top-k)
def test_topk_golden_rows():
    for ln in _lines("topk_rows.txt"):
        k, p, kept = (part.strip() for part in ln.split("|"))
        keep, _ = oracle.select_topk_row(np.array([float(x) for x in p.split()]), int(k))
        assert np.nonzero(keep)[0].tolist() == [int(x) for x in kept.split()], ln


def test_topk_invariants_on_random_rows():
    """Exactly min(k, n) kept; every kept probability >= every dropped one;
    at the cut, an equal probability is kept only if every lower index with
    that probability is kept too; k = 1 is numpy's argmax (first maximum)."""
    rng = np.random.default_rng(5)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        # coarse values so that ties are common
        p = rng.integers(0, 6, n).astype(np.float64)
        p = p / max(p.sum(), 1.0)
        for k in (1, 2, n // 2, n - 1, n, n + 3):
            if k < 1:
                continue
            keep, diag = oracle.select_topk_row(p, k)
            kept, dropped = p[keep == 1], p[keep == 0]
            assert keep.sum() == min(k, n)
            if dropped.size and kept.size:
                assert kept.min() >= dropped.max()
                cut = kept.min()
                tied = np.nonzero(p == cut)[0]
                flags = keep[tied]
                assert np.all(np.diff(flags.astype(int)) <= 0), "a higher index won a tie"
                assert diag[0] == cut and diag[1] == dropped.max()
            if k == 1:
                assert np.nonzero(keep)[0].tolist() == [int(np.argmax(p))]


def test_topk_agrees_with_topp_prefix():
    """Top-p keeps a prefix of the same (probability desc, index asc) order, so
    top-k with k = the top-p count must keep the same set."""
    wl = workloads.get("tiny")
    q, k, _ = workloads.make_qkv(wl)
    qf, kf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k))
    qp, kp = oracle.pool(qf), oracle.pool(kf)
    keep_p, _ = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, 0.2, False)
    counts = keep_p.sum(axis=1)
    for kk in np.unique(counts):
        rows = np.nonzero(counts == kk)[0]
        keep_k, _ = oracle.block_mask_topk(qp, kp, wl.Hb, wl.Wb, int(kk), False, rows=rows)
        np.testing.assert_array_equal(keep_k, keep_p[rows])


def test_sta_mask_closed_form_and_fixture():
    """Row counts are products of clipped window widths; the mask is symmetric;
    radius 0 is the identity; it agrees with the hand-derived window fixture."""
    for T, Hb, Wb, rad in [(3, 3, 3, (1, 1, 1)), (4, 2, 5, (0, 1, 2)), (2, 3, 4, (0, 0, 0)),
                           (5, 4, 6, (2, 1, 1)), (2, 2, 2, (9, 9, 9))]:
        m = oracle.sta_mask(T, Hb, Wb, rad)
        Nb = T * Hb * Wb
        r = np.arange(Nb)
        t, y, x = r // (Hb * Wb), (r // Wb) % Hb, r % Wb

        def span(c, rr, n):
            return np.minimum(c + rr, n - 1) - np.maximum(c - rr, 0) + 1
        want = span(t, rad[0], T) * span(y, rad[1], Hb) * span(x, rad[2], Wb)
        np.testing.assert_array_equal(m.sum(axis=1), want)
        np.testing.assert_array_equal(m, m.T)
        if rad == (0, 0, 0):
            np.testing.assert_array_equal(m, np.eye(Nb, dtype=np.uint8))
    # the fixture lists the window of given rows on a 3x3x3 grid, radius 1
    m = oracle.sta_mask(3, 3, 3, (1, 1, 1))
    for ln in _lines("sta_window_T3_Hb3_Wb3_r1.txt"):
        r, cols = (part.strip() for part in ln.split(":"))
        assert np.nonzero(m[int(r)])[0].tolist() == [int(c) for c in cols.split()], ln


# ---------------------------------------------------------------- f4 query subset
def test_query_subset_rows_equal_full_rows_and_dense():
    """Attention restricted to listed query blocks gives exactly those rows of
    the full result; with every block kept they are rows of textbook dense
    attention (torch SDPA in fp64)."""
    wl = workloads.get("tiny")
    q, k, v = workloads.make_qkv(wl)
    qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
    rows = wl.B * wl.heads * wl.Nb
    keep = np.ones((rows, wl.Nb), dtype=np.uint8)
    rp, ci = oracle.mask_to_csr(keep)
    o_all, l_all = oracle.sparse_attention(qf, kf, vf, rp, ci)
    sub = np.array([0, 3, 5, 16, 17, 31])
    o_sub, l_sub = oracle.sparse_attention(qf, kf, vf, rp, ci, qblocks=sub)
    idx = (sub[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
    np.testing.assert_array_equal(o_sub, o_all[idx])
    np.testing.assert_array_equal(l_sub, l_all[idx])
    qt, kt, vt = (oracle.to_bf16_tensor(x).double() for x in (qf, kf, vf))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    np.testing.assert_allclose(o_sub, ref.reshape(-1, wl.d).numpy()[idx], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- f1 semantic-aware permutation
def _bf16_u16(a: np.ndarray) -> np.ndarray:
    return oracle.as_u16(torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16))


def test_kmeans_recovers_planted_clusters():
    """Three well-separated groups laid out so that the evenly spaced initial
    tokens fall one in each: labels recover the groups and centroids are the
    groups' means."""
    rng = np.random.default_rng(8)
    d, n = 16, 90
    centers = np.zeros((3, d))
    centers[0, 0], centers[1, 1], centers[2, 2] = 20.0, -20.0, 20.0
    truth = np.arange(n) % 3
    x = _bf16_u16(centers[truth] + 0.1 * rng.standard_normal((n, d)))
    # group-major layout: the initial tokens 0, 30, 60 fall one per group
    order = np.argsort(truth, kind="stable")            # 0..0 1..1 2..2
    xs = x[order]
    label, cent, count = oracle.kmeans(xs, 3, 4)
    np.testing.assert_array_equal(label, np.repeat([0, 1, 2], n // 3))
    np.testing.assert_array_equal(count, [n // 3] * 3)
    xf = oracle.to_f64(xs)
    for j in range(3):
        np.testing.assert_allclose(cent[j], xf[label == j].mean(axis=0), rtol=1e-6, atol=1e-6)


def test_kmeans_assign_is_argmin_of_numpy_distances():
    """The oracle's ||c~||^2 - 2 x.c~ against numpy's full squared distance
    with the same bf16-rounded centroids; ties would go to the lower index in
    both (numpy argmin returns the first minimum)."""
    rng = np.random.default_rng(9)
    x = _bf16_u16(rng.standard_normal((200, 32)))
    cent = rng.standard_normal((7, 32)).astype(np.float32)
    label, diag = oracle.kmeans_assign(x, cent)
    cb = oracle.to_f64(_bf16_u16(cent))
    dist = ((oracle.to_f64(x)[:, None, :] - cb[None, :, :]) ** 2).sum(-1)
    np.testing.assert_array_equal(label, np.argmin(dist, axis=1))
    xn = (oracle.to_f64(x) ** 2).sum(-1)
    np.testing.assert_allclose(diag[:, 0] + xn, dist.min(axis=1), rtol=1e-12, atol=1e-9)


def test_kmeans_update_means_and_empty_cluster():
    rng = np.random.default_rng(10)
    x = _bf16_u16(rng.standard_normal((50, 8)))
    label = rng.integers(0, 3, 50).astype(np.int32)          # cluster 3 is empty
    old = rng.standard_normal((4, 8)).astype(np.float32)
    cent, count = oracle.kmeans_update(x, label, old)
    np.testing.assert_array_equal(count, np.bincount(label, minlength=4))
    xf = oracle.to_f64(x)
    for j in range(3):
        np.testing.assert_allclose(cent[j], xf[label == j].mean(axis=0).astype(np.float32),
                                   rtol=0, atol=2e-7)
    np.testing.assert_array_equal(cent[3], old[3])


def test_cluster_order_is_stable_sort():
    rng = np.random.default_rng(12)
    label = rng.integers(0, 9, 500).astype(np.int32)
    order, start = oracle.cluster_order(label, 10)
    np.testing.assert_array_equal(order, np.argsort(label, kind="stable"))
    np.testing.assert_array_equal(start, np.concatenate([[0], np.cumsum(np.bincount(label, minlength=10))]))


def test_centroid_topp_size_weighting():
    """Two key clusters with the same centroid: estimated attention in the
    ratio of their sizes (30:10, so 0.75 and 0.25 exactly); an empty cluster
    gets none."""
    ck = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 5.0]], dtype=np.float32)
    cq = np.array([[0.5, 0.0]], dtype=np.float32)
    nk = np.array([30, 10, 0], dtype=np.int32)
    keep, diag = oracle.centroid_topp(cq, ck, nk, 0.75)       # 0.75 = 30/40 exactly
    np.testing.assert_array_equal(keep[0], [1, 0, 0])
    keep, _ = oracle.centroid_topp(cq, ck, nk, 0.8)
    np.testing.assert_array_equal(keep[0], [1, 1, 0])
    # p = 1 keeps every cluster, as thr = 0 does in the top-p rule (an empty
    # cluster brings no keys)
    keep, _ = oracle.centroid_topp(cq, ck, nk, 1.0)
    np.testing.assert_array_equal(keep[0], [1, 1, 1])


def test_centroid_topp_scale_is_inverse_sqrt_d():
    """Two equal-size key clusters with opposite centroids: the estimated
    attention of the first is the logistic function of the score difference
    2a/sqrt(d) (a = ln 3, d = 4 gives exactly 3/4 in exact arithmetic).  A
    dropped or doubled scale would give logistic(2a) = 0.9, a factor sqrt(d)
    in place of 1/sqrt(d) gives 81/82."""
    d = 4
    a = np.float32(np.log(3.0))
    cq = np.zeros((1, d), dtype=np.float32)
    cq[0, 0] = a
    ck = np.zeros((2, d), dtype=np.float32)
    ck[0, 0], ck[1, 0] = 1.0, -1.0
    nk = np.array([7, 7], dtype=np.int32)
    p0 = 1.0 / (1.0 + np.exp(-2.0 * float(a) / np.sqrt(d)))       # ~0.75
    keep, diag = oracle.centroid_topp(cq, ck, nk, 0.74)
    np.testing.assert_array_equal(keep[0], [1, 0])
    np.testing.assert_allclose(diag[0, 2], p0, rtol=1e-14)         # last kept probability
    np.testing.assert_allclose(diag[0, 3], 1.0 - p0, rtol=1e-14)   # first dropped
    keep, _ = oracle.centroid_topp(cq, ck, nk, 0.76)               # 0.75 < 0.76: both
    np.testing.assert_array_equal(keep[0], [1, 1])


def test_cluster_attention_against_masked_sdpa_and_permutation():
    """Token-level attention over kept clusters equals torch SDPA with the
    boolean mask built from the labels; all clusters kept is dense attention;
    and computing it on the permuted sequence and permuting back gives the
    same result (SVG2 section 2A)."""
    wl = workloads.get("tiny")
    q, k, v = workloads.make_qkv(wl)
    qu, ku, vu = (oracle.as_u16(x)[0, 0] for x in (q, k, v))
    lq, cq, nq = oracle.kmeans(qu, 6, 2)
    lk, ck, nk = oracle.kmeans(ku, 9, 2)
    keep, _ = oracle.centroid_topp(cq, ck, nk, 0.7)
    tok = np.arange(wl.N)
    o, lse = oracle.cluster_attention(qu, ku, vu, lq, lk, keep, tok)
    qt, kt, vt = (torch.from_numpy(oracle.to_f64(x)) for x in (qu, ku, vu))
    mask = torch.from_numpy(keep[lq][:, lk].astype(bool))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    ones = np.ones_like(keep)
    o_all, _ = oracle.cluster_attention(qu, ku, vu, lq, lk, ones, tok)
    dense = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    np.testing.assert_allclose(o_all, dense.numpy(), rtol=0, atol=1e-12)
    # permuted computation, permuted back
    oq, _ = oracle.cluster_order(lq, 6)
    ok, _ = oracle.cluster_order(lk, 9)
    pm = torch.from_numpy(keep[lq[oq]][:, lk[ok]].astype(bool))
    perm = torch.nn.functional.scaled_dot_product_attention(qt[oq], kt[ok], vt[ok], attn_mask=pm)
    back = torch.empty_like(perm)
    back[torch.from_numpy(oq)] = perm
    np.testing.assert_allclose(back.numpy(), o, rtol=0, atol=1e-12)
