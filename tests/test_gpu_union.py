"""GPU parity of band-plus-shared-window attention (spa_attn_fwd_union /
spa_attn_bwd_union through the C ABI) against the fp64 oracle's union
entries, on the same seeded bf16 inputs.  Tolerances as in
test_gpu_parity.py: |o - o_ref| <= 2e-2, |lse - lse_ref| <= 1e-3, each
gradient max-abs error <= 5e-2 of the reference's max-abs value."""
import math

import numpy as np
import pytest
import torch

import oracle
from head_partitioned_distance_b200 import synth

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL = 2e-2, 1e-3, 5e-2


@pytest.fixture(scope="module")
def spa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from head_partitioned_distance_b200 import spa as mod
    return mod


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _check_grad(g, ref, name):
    assert not np.isnan(g).any(), name
    err = np.abs(g - ref).max()
    assert err / np.abs(ref).max() <= GRAD_TOL, (name, err)


def _gpu(spa, q, k, v, do, scale, window, lo=None, hi=None):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = spa.attention_forward_union(qd, kd, vd, window, scale, lo, hi)
    dq, dk, dv = spa.attention_backward_union(qd, kd, vd, o, dod, lse, window, scale, lo, hi)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    return {n: _f64(t) for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}


CASES = [
    (1, 4, 600, 64, 1),      # window = the diagonal only
    (1, 4, 600, 64, 100),    # window apart from every band but head 0's
    (1, 4, 600, 64, 200),    # window overlapping head 1's band
    (1, 4, 600, 64, 600),    # window covering every distance: dense causal
    (2, 5, 777, 128, 37),
    (1, 8, 1001, 64, 64),
    (1, 3, 129, 128, 5),
    (1, 32, 2048, 128, 256),
    # both parts at least 768 wide on average: the merging forward in the
    # form whose softmax warpgroups take turns
    (1, 1, 2000, 64, 10),
    (2, 2, 3200, 128, 700),
]


@pytest.mark.parametrize("B,H,N,d,w", CASES)
def test_union_every_element(spa, B, H, N, d, w):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=101 + N + w)
    scale = 1 / math.sqrt(d)
    got = _gpu(spa, q, k, v, do, scale, w)
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.union_fwd(qf, kf, vf, scale, w)
    assert np.isfinite(got["lse"]).all()  # distance 0 is in every set
    assert np.abs(got["o"] - o_ref).max() <= O_TOL
    assert np.abs(got["lse"] - lse_ref).max() <= LSE_TOL
    for name, ref in zip(("dq", "dk", "dv"), oracle.union_bwd(qf, kf, vf, dof, scale, w)):
        _check_grad(got[name], ref, name)


def test_union_autograd_function(spa):
    B, H, N, d, w = 1, 8, 1001, 64, 64
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=211)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    o = spa.spattention_union(qd, kd, vd, w)
    o.backward(do.to(dev))
    scale = d ** -0.5
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, _ = oracle.union_fwd(qf, kf, vf, scale, w)
    assert np.abs(_f64(o) - o_ref).max() <= O_TOL
    for g, ref, name in zip((qd.grad, kd.grad, vd.grad), oracle.union_bwd(qf, kf, vf, dof, scale, w), "qkv"):
        _check_grad(_f64(g), ref, name)


def test_union_with_explicit_bands(spa):
    B, H, N, d, w = 1, 4, 600, 64, 50
    lo, hi = [0, 3, 257, 40], [1, 400, 300, 600]
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=77)
    got = _gpu(spa, q, k, v, do, 0.125, w, lo, hi)
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.union_fwd(qf, kf, vf, 0.125, w, np.array(lo), np.array(hi))
    assert np.abs(got["o"] - o_ref).max() <= O_TOL
    assert np.abs(got["lse"] - lse_ref).max() <= LSE_TOL
    refs = oracle.union_bwd(qf, kf, vf, dof, 0.125, w, np.array(lo), np.array(hi))
    for name, ref in zip(("dq", "dk", "dv"), refs):
        _check_grad(got[name], ref, name)


def test_union_full_size_sampled_rows(spa):
    # the benchmark's union workload: B1 H32 N32768 d128, window 256
    w = synth.WORKLOADS["b1_h32_n32768_d128"]
    window = 256
    q, k, v, do = synth.workload_inputs(w)
    got = _gpu(spa, q, k, v, do, w.scale, window)
    B, H, N, d = w.B, w.H, w.N, w.d
    lo, hi = oracle.bands(N, H)
    per_head = [[0, window - 1, window, int(lo[h]), int(lo[h]) + 1, N - 1] for h in range(H)]
    rows = synth.sample_rows(B, H, N, 32, seed=w.seed + 7, per_head=per_head)
    key_rows = [N - 1, 0, window, (H - 1) * N + N - 1 - int(lo[H - 1]), 5 * N + 1000]
    flat = lambda x: x.reshape(B * H * N, -1)
    res = {n: ([], []) for n in ("o", "lse", "dq", "dk", "dv")}
    for bh in sorted(set(r // N for r in rows) | set(r // N for r in key_rows)):
        h = bh % H
        sl = lambda t: _f64(t.reshape(B * H, N, d)[bh])[None, None]
        qh, kh, vh, doh = sl(q), sl(k), sl(v), sl(do)
        blo, bhi = lo[h:h + 1], hi[h:h + 1]
        rs = [r % N for r in rows if r // N == bh]
        if rs:
            o_r, l_r = oracle.union_fwd_rows(qh, kh, vh, w.scale, window, rs, blo, bhi)
            dq_r = oracle.union_bwd_dq_rows(qh, kh, vh, doh, w.scale, window, rs, blo, bhi)
            idx = [bh * N + i for i in rs]
            for n, g, r in (("o", flat(got["o"])[idx], o_r), ("dq", flat(got["dq"])[idx], dq_r),
                            ("lse", got["lse"].reshape(-1)[idx], l_r)):
                res[n][0].append(g)
                res[n][1].append(r)
        ks = [r % N for r in key_rows if r // N == bh]
        if ks:
            dk_r, dv_r = oracle.union_bwd_dkdv_rows(qh, kh, vh, doh, w.scale, window, ks, blo, bhi)
            idx = [bh * N + j for j in ks]
            for n, g, r in (("dk", flat(got["dk"])[idx], dk_r), ("dv", flat(got["dv"])[idx], dv_r)):
                res[n][0].append(g)
                res[n][1].append(r)
    cat = lambda xs: np.concatenate(xs, axis=0)
    assert np.abs(cat(res["o"][0]) - cat(res["o"][1])).max() <= O_TOL
    assert np.abs(cat(res["lse"][0]) - cat(res["lse"][1])).max() <= LSE_TOL
    for name in ("dq", "dk", "dv"):
        _check_grad(cat(res[name][0]), cat(res[name][1]), name)


def test_launch_by_launch_composition_equals_the_union_calls(spa):
    # spa_union_parts + the band forward, the merging forward and the adding
    # backward passes, called one by one, are exactly what the two union
    # calls launch; merging / summing part 2 computed into separate buffers
    # (spa_attn_union_merge, spa_attn_union_add_grads) agrees to bf16 rounding
    B, H, N, d, w = 1, 8, 1001, 64, 64
    q, k, v, do = (t.to("cuda:0") for t in synth.make_inputs(B, H, N, d, seed=5))
    scale = 0.125
    o, lse = spa.attention_forward_union(q, k, v, w, scale)
    dq, dk, dv = spa.attention_backward_union(q, k, v, o, do, lse, w, scale)
    a1, b1, a2, b2 = spa.spa_union_parts(N, H, w)
    o1, l1 = spa.attention_forward(q, k, v, scale, a1, b1)
    om, lm = o1.clone(), l1.clone()
    spa.spa_attn_fwd_merge(q, k, v, o1, l1, scale, a2, b2)
    o2, l2 = spa.attention_forward(q, k, v, scale, a2, b2)
    spa.spa_attn_union_merge(om, lm, o2, l2)
    ws = torch.empty(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device="cuda:0")
    g1 = [torch.empty_like(q) for _ in range(3)]
    spa.spa_attn_bwd_dq_delta(q, k, v, o1, do, l1, ws, g1[0], scale, a1, b1)
    spa.spa_attn_bwd_dkdv(q, k, v, do, l1, ws, g1[1], g1[2], scale, a1, b1)
    g2 = [t.clone() for t in g1]
    spa.spa_attn_bwd_dq_add(q, k, v, do, l1, ws, g1[0], scale, a2, b2)
    spa.spa_attn_bwd_dkdv_add(q, k, v, do, l1, ws, g1[1], g1[2], scale, a2, b2)
    p2 = [torch.empty_like(q) for _ in range(3)]
    spa.spa_attn_bwd_dq(q, k, v, do, l1, ws, p2[0], scale, a2, b2)
    spa.spa_attn_bwd_dkdv(q, k, v, do, l1, ws, p2[1], p2[2], scale, a2, b2)
    spa.spa_attn_union_add_grads(*g2, *p2)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    assert torch.equal(o, o1) and torch.equal(lse, l1)
    # merged in the epilogue vs merged from two bf16 outputs: two roundings against one
    assert (o.float() - om.float()).abs().max() <= 2 ** -7 * o.float().abs().max()
    assert (lse - lm).abs().max() <= 1e-4
    for a, b, c in zip((dq, dk, dv), g1, g2):
        assert torch.equal(a, b)
        # two roundings (part 2 to bf16, then the sum) against one
        assert (a.float() - c.float()).abs().max() <= 2 ** -7 * a.float().abs().max()


@pytest.mark.parametrize("B,H,N,d", [(1, 4, 600, 64), (2, 3, 777, 128)])
def test_split_bands_merge_and_add_to_the_whole_band(spa, B, H, N, d):
    # every head's band [lo, hi) cut at an arbitrary distance m into [lo, m)
    # and [m, hi): the forward of the first part then the merging forward of
    # the second give the whole band's o and lse, and the backward passes of
    # the first part then the adding passes of the second (with the whole
    # band's lse and D) give its gradients; rows the second part leaves empty
    # (i < m) keep the first part's values
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=17 + N)
    scale = 1 / math.sqrt(d)
    lo, hi = oracle.bands(N, H)
    cut = [int(a + (b - a) // 3 + 1) for a, b in zip(lo, hi)]
    lo1, hi1 = [int(x) for x in lo], cut
    lo2, hi2 = cut, [int(x) for x in hi]
    qd, kd, vd, dod = (t.to("cuda:0") for t in (q, k, v, do))
    o, lse = spa.attention_forward(qd, kd, vd, scale, lo1, hi1)
    spa.spa_attn_fwd_merge(qd, kd, vd, o, lse, scale, lo2, hi2)
    ws = torch.empty(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device="cuda:0")
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    spa.spa_attn_bwd_dq_delta(qd, kd, vd, o, dod, lse, ws, dq, scale, lo1, hi1)
    spa.spa_attn_bwd_dkdv(qd, kd, vd, dod, lse, ws, dk, dv, scale, lo1, hi1)
    spa.spa_attn_bwd_dq_add(qd, kd, vd, dod, lse, ws, dq, scale, lo2, hi2)
    spa.spa_attn_bwd_dkdv_add(qd, kd, vd, dod, lse, ws, dk, dv, scale, lo2, hi2)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.spa_fwd(qf, kf, vf, scale)
    got_lse = _f64(lse)
    neg = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(got_lse), neg)
    assert np.abs(_f64(o) - o_ref).max() <= O_TOL
    assert np.abs(got_lse[~neg] - lse_ref[~neg]).max() <= LSE_TOL
    for name, g, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), oracle.spa_bwd(qf, kf, vf, dof, scale)):
        _check_grad(_f64(g), ref, name)
