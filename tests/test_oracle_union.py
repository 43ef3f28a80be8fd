"""Pins for the oracle's band-plus-shared-window attention (each head attends
to its band [lo_h, hi_h) and to the distances [0, w) that every head shares;
a reading of the local sharing that the EBALL ablation of "Making Every Head
Count", Figure 2(b), takes out).  The checks reduce it to the band
oracle (w = 0), to dense causal attention (w >= N), to torch's fp64
scaled_dot_product_attention with the union written as an explicit mask
(forward and autograd backward), and to the log-sum-exp merge of its two
disjoint parts."""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _union_mask(N, w, lo, hi):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    dist = i - j
    return (j <= i) & ((dist < w) | ((dist >= lo) & (dist < hi)))


def _sdpa(q, k, v, mask, scale):
    qt, kt, vt = (torch.from_numpy(x) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale).numpy()


def test_zero_window_is_the_band():
    B, H, N, d = 2, 4, 37, 6
    q, k, v, do = (_rand((B, H, N, d), s) for s in (1, 2, 3, 4))
    o, lse = oracle.union_fwd(q, k, v, 0.4, 0)
    ob, lb = oracle.spa_fwd(q, k, v, 0.4)
    np.testing.assert_allclose(o, ob, atol=1e-13, rtol=0)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-13, rtol=0)
    for a, b in zip(oracle.union_bwd(q, k, v, do, 0.4, 0), oracle.spa_bwd(q, k, v, do, 0.4)):
        np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def test_window_covering_every_distance_is_dense_causal():
    B, H, N, d = 1, 3, 29, 5
    q, k, v = (_rand((B, H, N, d), s) for s in (5, 6, 7))
    o, _ = oracle.union_fwd(q, k, v, 0.7, N)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), is_causal=True, scale=0.7).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("N,H,w", [(41, 5, 3), (64, 4, 20), (50, 7, 1), (33, 3, 12)])
def test_each_head_is_masked_dense_attention(N, H, w):
    B, d = 2, 8
    q, k, v, do = (_rand((B, H, N, d), s) for s in (8 + w, 9 + w, 10 + w, 11 + w))
    scale = 1 / math.sqrt(d)
    o, lse = oracle.union_fwd(q, k, v, scale, w)
    dq, dk, dv = oracle.union_bwd(q, k, v, do, scale, w)
    lo, hi = oracle.bands(N, H)
    for h in range(H):
        m = _union_mask(N, w, lo[h], hi[h])
        assert m.any(axis=1).all()  # distance 0 is in every set when w >= 1
        np.testing.assert_allclose(o[:, h], _sdpa(q[:, h], k[:, h], v[:, h], m, scale), atol=1e-12, rtol=0)
        s = scale * np.einsum("bid,bjd->bij", q[:, h], k[:, h])
        ref_lse = torch.logsumexp(torch.from_numpy(np.where(m, s, -np.inf)), -1).numpy()
        np.testing.assert_allclose(lse[:, h], ref_lse, atol=1e-12, rtol=0)
        qt, kt, vt = (torch.tensor(x[:, h], requires_grad=True) for x in (q, k, v))
        out = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(m), scale=scale)
        (out * torch.from_numpy(do[:, h])).sum().backward()
        np.testing.assert_allclose(dq[:, h], qt.grad.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dk[:, h], kt.grad.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dv[:, h], vt.grad.numpy(), atol=1e-12, rtol=0)


def test_disjoint_parts_merge_through_their_lse():
    # w <= lo_h on every head but the first: the set is the disjoint union of
    # [0, w) and the band, and softmax over it is the lse-weighted mix of the
    # two partial softmaxes (a property of exp, not of this code)
    B, H, N, d = 1, 4, 48, 5
    q, k, v = (_rand((B, H, N, d), s) for s in (12, 13, 14))
    w = 5
    lo, hi = oracle.bands(N, H)  # lo = 0, 12, 24, 36
    o, lse = oracle.union_fwd(q, k, v, 0.6, w)
    o1, l1 = oracle.spa_fwd(q, k, v, 0.6, lo=[0] * H, hi=[w] * H)
    o2, l2 = oracle.spa_fwd(q, k, v, 0.6, lo=lo, hi=hi)
    for h in range(1, H):
        L = np.logaddexp(l1[0, h], l2[0, h])
        np.testing.assert_allclose(lse[0, h], L, atol=1e-12, rtol=0)
        w1 = np.exp(l1[0, h] - L)[:, None]
        w2 = np.where(np.isneginf(l2[0, h]), 0.0, np.exp(l2[0, h] - L))[:, None]
        np.testing.assert_allclose(o[0, h], w1 * o1[0, h] + w2 * o2[0, h], atol=1e-12, rtol=0)


def test_row_entries_match_full_tensor():
    B, H, N, d = 2, 3, 40, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (15, 16, 17, 18))
    o, lse = oracle.union_fwd(q, k, v, 0.5, 7)
    dq, dk, dv = oracle.union_bwd(q, k, v, do, 0.5, 7)
    rows = list(range(0, B * H * N, 5)) + [B * H * N - 1]
    flat = lambda t: t.reshape(B * H * N, -1)
    orow, lrow = oracle.union_fwd_rows(q, k, v, 0.5, 7, rows)
    np.testing.assert_array_equal(orow, flat(o)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])
    np.testing.assert_allclose(oracle.union_bwd_dq_rows(q, k, v, do, 0.5, 7, rows), flat(dq)[rows],
                               atol=1e-12, rtol=0)
    dkr, dvr = oracle.union_bwd_dkdv_rows(q, k, v, do, 0.5, 7, rows)
    np.testing.assert_allclose(dkr, flat(dk)[rows], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dvr, flat(dv)[rows], atol=1e-12, rtol=0)
