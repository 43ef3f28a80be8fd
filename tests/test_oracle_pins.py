"""Pins for the fp64 CPU oracle: values the pages print, closed forms,
invariants, special cases that reduce to library routines, and finite
differences.  None of these compare the oracle with itself."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from head_partitioned_distance_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_sections(path):
    sections, cur = {}, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = line.strip("[]")
                sections[cur] = []
            else:
                sections[cur].append(line)
    return sections


# ---------------------------------------------------------------------------
# (a) generic masked softmax: the worked example of "Story of Attention --
#     Part 4", section 1 (Sparse Transformer), subsection "Worked example".
# ---------------------------------------------------------------------------
def _worked_example():
    s = _read_sections(os.path.join(GOLDEN, "worked_example_strided_4x4.txt"))
    mat = {k: np.array([[float(x) for x in row.split()] for row in v]) for k, v in s.items()}
    return mat


def test_worked_example_scores_exact():
    m = _worked_example()
    scores, attn, o, lse = oracle.masked_attn_fwd(m["Q"], m["K"], m["V"], m["MASK"], 0.5)
    # scores are scale * Q K^T with scale 1/2: exact in fp64 for these integers
    np.testing.assert_array_equal(scores / 0.5, m["QKT"])


def test_worked_example_attention_and_output():
    m = _worked_example()
    _, attn, o, lse = oracle.masked_attn_fwd(m["Q"], m["K"], m["V"], m["MASK"], 0.5)
    # masked entries are exactly zero, permitted ones match the printed A
    assert np.all(attn[m["MASK"] == 0] == 0.0)
    np.testing.assert_allclose(attn, m["A"], atol=5e-4, rtol=0)
    # rows of A sum to one over the permitted set
    np.testing.assert_allclose(attn.sum(axis=1), 1.0, atol=1e-15)
    expected = m["OUTPUT"].copy()
    # The page multiplied its rounded A by V for the last entry (0.622 * 5);
    # check that reading, then the exact entry against the exact weight.
    assert abs(np.round(attn, 3)[3] @ m["V"][:, 3] - expected[3, 3]) < 5e-4
    exact_44 = 5.0 / (1.0 + math.exp(-0.5))  # weight of key 4 in row 4, times v = 5
    assert abs(o[3, 3] - exact_44) < 1e-12
    expected[3, 3] = exact_44
    np.testing.assert_allclose(o, expected, atol=5e-4, rtol=0)


def test_worked_example_single_key_rows_copy_value():
    # rows 1 and 2 see one key each: weight 1, output = that value row,
    # lse = its scaled score
    m = _worked_example()
    _, attn, o, lse = oracle.masked_attn_fwd(m["Q"], m["K"], m["V"], m["MASK"], 0.5)
    np.testing.assert_array_equal(o[0], m["V"][0])
    np.testing.assert_array_equal(o[1], m["V"][1])
    assert lse[0] == 0.5 * m["QKT"][0, 0] and lse[1] == 0.5 * m["QKT"][1, 1]


# ---------------------------------------------------------------------------
# (b) Balanced Distance Partitioning: complete, exclusive, balanced bands,
#     head 0 nearest ("Making Every Head Count", Figure 1 caption; TL;DR).
# ---------------------------------------------------------------------------
def _check_bands(N, H):
    lo, hi = oracle.bands(N, H)
    assert lo[0] == 0 and hi[-1] == N
    assert np.all(hi[:-1] == lo[1:])  # contiguous and non-overlapping
    widths = hi - lo
    assert set(widths.tolist()) <= {N // H, -(-N // H)}
    assert np.all(widths >= 1)
    assert np.all(np.diff(lo) > 0)  # head h+1 strictly farther than head h


def test_bands_invariants_sweep():
    for N in range(1, 161):
        for H in range(1, N + 1):
            _check_bands(N, H)
    for N, H in [(4096, 16), (8192, 32), (32768, 32), (30001, 32), (1001, 8),
                 (2 ** 31 - 1, 7), (10 ** 12 + 7, 64)]:
        _check_bands(N, H)


def test_bands_figure1_layout_and_workloads():
    lo, hi = oracle.bands(1024, 8)  # Figure 1: N=1024, H=8, eight width-128 bands
    assert lo.tolist() == [0, 128, 256, 384, 512, 640, 768, 896]
    assert (hi - lo).tolist() == [128] * 8
    lo, hi = oracle.bands(1001, 8)
    assert sorted(set((hi - lo).tolist())) == [125, 126]
    lo, hi = oracle.bands(1000, 8)
    assert set((hi - lo).tolist()) == {125}
    lo, hi = oracle.bands(30001, 32)
    assert sorted(set((hi - lo).tolist())) == [937, 938]


def test_bands_reject_bad_requests():
    for N, H in [(0, 1), (5, 0), (3, 4)]:
        with pytest.raises(ValueError):
            oracle.bands(N, H)


def test_pair_count_is_one_causal_attention():
    # The H heads together cover every causal pair once: N(N+1)/2 per batch.
    for N in list(range(1, 40)) + [64, 100, 129]:
        for H in range(1, N + 1):
            lo, hi = oracle.bands(N, H)
            per_head = [oracle.band_pairs(N, int(a), int(b)) for a, b in zip(lo, hi)]
            assert sum(per_head) == N * (N + 1) // 2
            # closed form per head: distance delta occurs in N - delta rows
            for (a, b), p in zip(zip(lo, hi), per_head):
                assert p == sum(N - dd for dd in range(int(a), int(b)))


def test_workload_pair_counts():
    for name, w in synth.WORKLOADS.items():
        if w.N > 4096:
            continue  # one-by-one count is quadratic; the closed form is checked above
        lo, hi = oracle.bands(w.N, w.H)
        pairs = sum(oracle.band_pairs(w.N, int(a), int(b)) for a, b in zip(lo, hi))
        assert w.B * pairs == w.B * w.N * (w.N + 1) // 2


# ---------------------------------------------------------------------------
# (c) special cases that reduce to textbook attention
# ---------------------------------------------------------------------------
def _rand(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    mt = None if mask is None else torch.from_numpy(mask.astype(bool))
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=mt, is_causal=causal, scale=scale).numpy()


def test_one_head_is_dense_causal_attention():
    B, H, N, d = 2, 1, 37, 8
    q, k, v = (_rand((B, H, N, d), s) for s in (1, 2, 3))
    o, lse = oracle.spa_fwd(q, k, v, 0.3)
    ref = _sdpa(q, k, v, causal=True, scale=0.3)
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)
    s = 0.3 * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(s), -1).numpy(),
                               atol=1e-12, rtol=0)


def test_full_band_on_every_head_is_dense_causal_per_head():
    B, H, N, d = 1, 3, 29, 5
    q, k, v = (_rand((B, H, N, d), s) for s in (4, 5, 6))
    o, _ = oracle.spa_fwd(q, k, v, 0.7, lo=[0] * H, hi=[N] * H)
    np.testing.assert_allclose(o, _sdpa(q, k, v, causal=True, scale=0.7), atol=1e-12, rtol=0)


def _band_mask(N, lo, hi):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    return (j <= i) & (i - j >= lo) & (i - j < hi)


@pytest.mark.parametrize("N,H", [(41, 5), (64, 4), (33, 33), (50, 7)])
def test_each_head_is_masked_dense_attention(N, H):
    B, d = 2, 16
    q, k, v = (_rand((B, H, N, d), s) for s in (7, 8, 9))
    scale = 1 / math.sqrt(d)
    o, lse = oracle.spa_fwd(q, k, v, scale)
    lo, hi = oracle.bands(N, H)
    for h in range(H):
        mask = _band_mask(N, lo[h], hi[h])
        rows = mask.any(axis=1)
        assert np.all(rows == (np.arange(N) >= lo[h]))
        mfix = mask.copy()
        mfix[~rows] = True  # SDPA needs a non-empty set; these rows are checked separately
        ref = _sdpa(q[:, h], k[:, h], v[:, h], mask=mfix, scale=scale)
        np.testing.assert_allclose(o[:, h][:, rows], ref[:, rows], atol=1e-12, rtol=0)
        # empty-band convention: zero output, lse = -inf
        assert np.all(o[:, h][:, ~rows] == 0.0)
        assert np.all(np.isneginf(lse[:, h][:, ~rows]))
        assert np.all(np.isfinite(lse[:, h][:, rows]))


def test_one_distance_per_head_copies_value_rows():
    # H = N: head h sees exactly the key at distance h, so o_i = v_{i-h} and
    # lse_i = scale * q_i . k_{i-h} (softmax over one element).
    N = H = 9
    d = 4
    q, k, v = (_rand((1, H, N, d), s) for s in (10, 11, 12))
    o, lse = oracle.spa_fwd(q, k, v, 0.5)
    for h in range(H):
        for i in range(N):
            if i < h:
                assert np.all(o[0, h, i] == 0) and np.isneginf(lse[0, h, i])
            else:
                np.testing.assert_array_equal(o[0, h, i], v[0, h, i - h])
                assert lse[0, h, i] == pytest.approx(0.5 * q[0, h, i] @ k[0, h, i - h], abs=1e-14)


def test_generic_masked_entry_matches_band_entry():
    N, H, d = 23, 4, 6
    q, k, v, do = (_rand((1, H, N, d), s) for s in (13, 14, 15, 16))
    o, lse = oracle.spa_fwd(q, k, v, 0.4)
    dq, dk, dv = oracle.spa_bwd(q, k, v, do, 0.4)
    lo, hi = oracle.bands(N, H)
    for h in range(H):
        m = _band_mask(N, lo[h], hi[h])
        _, _, og, lg = oracle.masked_attn_fwd(q[0, h], k[0, h], v[0, h], m, 0.4)
        np.testing.assert_allclose(og, o[0, h], atol=1e-13, rtol=0)
        np.testing.assert_allclose(lg, lse[0, h], atol=1e-13, rtol=0)
        gq, gk, gv = oracle.masked_attn_bwd(q[0, h], k[0, h], v[0, h], m, 0.4, do[0, h])
        for a, b in ((gq, dq), (gk, dk), (gv, dv)):
            np.testing.assert_allclose(a, b[0, h], atol=1e-12, rtol=0)


def test_row_entries_match_full_tensor_entries():
    B, H, N, d = 2, 3, 40, 8
    q, k, v, do = (_rand((B, H, N, d), s) for s in (17, 18, 19, 20))
    o, lse = oracle.spa_fwd(q, k, v, 0.35)
    dq, dk, dv = oracle.spa_bwd(q, k, v, do, 0.35)
    rows = list(range(0, B * H * N, 7)) + [B * H * N - 1]
    orow, lrow = oracle.spa_fwd_rows(q, k, v, 0.35, rows)
    flat = lambda t: t.reshape(B * H * N, -1)
    np.testing.assert_array_equal(orow, flat(o)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])
    np.testing.assert_allclose(oracle.spa_bwd_dq_rows(q, k, v, do, 0.35, rows), flat(dq)[rows],
                               atol=1e-12, rtol=0)
    dkr, dvr = oracle.spa_bwd_dkdv_rows(q, k, v, do, 0.35, rows)
    np.testing.assert_allclose(dkr, flat(dk)[rows], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dvr, flat(dv)[rows], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# (d) backward: torch autograd through SDPA, and central finite differences
# ---------------------------------------------------------------------------
def test_backward_matches_autograd_of_masked_sdpa():
    B, H, N, d = 1, 4, 30, 8
    q, k, v, do = (_rand((B, H, N, d), s) for s in (21, 22, 23, 24))
    scale = 0.45
    dq, dk, dv = oracle.spa_bwd(q, k, v, do, scale)
    lo, hi = oracle.bands(N, H)
    for h in range(H):
        m = _band_mask(N, lo[h], hi[h])
        rows = m.any(axis=1)
        mfix = m.copy()
        mfix[~rows] = True
        dof = do[:, h].copy()
        dof[:, ~rows] = 0.0  # empty rows contribute no gradient
        qt, kt, vt = (torch.tensor(x[:, h], requires_grad=True) for x in (q, k, v))
        out = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(mfix), scale=scale)
        (out * torch.from_numpy(dof)).sum().backward()
        np.testing.assert_allclose(dq[:, h], qt.grad.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dk[:, h], kt.grad.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dv[:, h], vt.grad.numpy(), atol=1e-12, rtol=0)


def test_backward_matches_central_finite_differences():
    B, H, N, d = 1, 3, 17, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (25, 26, 27, 28))
    scale = 0.6
    grads = oracle.spa_bwd(q, k, v, do, scale)

    def loss(qq, kk, vv):
        o, _ = oracle.spa_fwd(qq, kk, vv, scale)
        return float((o * do).sum())

    eps = 1e-6
    worst = 0.0
    for which in range(3):
        base = [q, k, v]
        g = grads[which]
        for idx in np.ndindex(*q.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            worst = max(worst, abs(fd - g[idx]))
        scale_g = np.abs(g).max()
        assert worst <= 1e-6 * max(scale_g, 1.0), (which, worst)


# ---------------------------------------------------------------------------
# tile classes: a hand-worked table, and the element mask summed per tile
# ---------------------------------------------------------------------------
def _hand_tile_cases():
    path = os.path.join(GOLDEN, "tile_classes_hand.txt")
    cases = []
    cur = None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("[case"):
                kv = dict(t.split("=") for t in line.strip("[]").split()[1:])
                cur = {"N": int(kv["N"]), "H": int(kv["H"]), "Bq": int(kv["Bq"]),
                       "Bk": int(kv["Bk"]), "heads": []}
                cases.append(cur)
            elif line.startswith("head"):
                cur["heads"].append([])
            else:
                cur["heads"][-1].append([int(x) for x in line.split()])
    return cases


def test_tile_classes_hand_worked():
    for c in _hand_tile_cases():
        lo, hi = oracle.bands(c["N"], c["H"])
        cls = oracle.tile_classes(c["N"], lo, hi, c["Bq"], c["Bk"])
        np.testing.assert_array_equal(cls, np.array(c["heads"], np.uint8))


@pytest.mark.parametrize("N,H,Bq,Bk", [(100, 4, 16, 8), (257, 3, 32, 64), (64, 64, 8, 8)])
def test_tile_classes_against_element_mask(N, H, Bq, Bk):
    lo, hi = oracle.bands(N, H)
    cls = oracle.tile_classes(N, lo, hi, Bq, Bk)
    nqt, nkt = -(-N // Bq), -(-N // Bk)
    for h in range(H):
        m = np.zeros((nqt * Bq, nkt * Bk), bool)
        m[:N, :N] = _band_mask(N, lo[h], hi[h])
        counts = m.reshape(nqt, Bq, nkt, Bk).sum(axis=(1, 3))
        want = np.where(counts == 0, 0, np.where(counts == Bq * Bk, 2, 1))
        np.testing.assert_array_equal(cls[h], want)
