"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle
on the same seeded bf16 inputs.

Tolerances (fp64 oracle as the truth):
  O                      max |o - o_ref|                      <= 2e-2
  lse (finite rows)      max |lse - lse_ref|                  <= 1e-3
  lse (empty rows)       exactly -inf where the oracle has -inf
  dq, dk, dv (each)      max |g - g_ref| / max |g_ref|        <= 5e-2
  NaN anywhere           failure
  tile classes           bit-exact
Small shapes compare every element; the full-size workloads compare sampled
rows that the oracle computes one by one (every head's first/last rows and
band edges, plus random rows)."""
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


def _gpu_run(spa, q, k, v, do, scale, lo=None, hi=None, backward=True, bwd="two-pass"):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = spa.attention_forward(qd, kd, vd, scale, lo, hi)
    out = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = spa.BACKWARDS[bwd](qd, kd, vd, o, dod, lse, scale, lo, hi)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    return {k_: _f64(v_) for k_, v_ in out.items()}


def _check_lse(lse, ref):
    neg = np.isneginf(ref)
    assert np.array_equal(np.isneginf(lse), neg), "empty-band rows must be exactly -inf"
    if (~neg).any():
        assert np.abs(lse[~neg] - ref[~neg]).max() <= LSE_TOL


# When the exact gradient is identically zero (a softmax over one key: dS =
# P (dO.v - D) = 0), the relative error is undefined; the bf16 rounding of o
# inside D leaves a residue of order 1e-7 * |dO| |v|, checked absolutely.
ZERO_GRAD_ABS_TOL = 1e-4


def _check_grad(g, ref, name):
    assert not np.isnan(g).any(), name
    denom = np.abs(ref).max()
    err = np.abs(g - ref).max()
    if denom == 0:
        assert err <= ZERO_GRAD_ABS_TOL, (name, err)
    else:
        assert err / denom <= GRAD_TOL, (name, err, denom)


def _full_check(spa, q, k, v, do, scale, lo=None, hi=None, bwd="two-pass"):
    got = _gpu_run(spa, q, k, v, do, scale, lo, hi, bwd=bwd)
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    lo_o = None if lo is None else np.array(lo)
    hi_o = None if hi is None else np.array(hi)
    o_ref, lse_ref = oracle.spa_fwd(qf, kf, vf, scale, lo_o, hi_o)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert not np.isnan(got[name]).any(), name
    assert np.abs(got["o"] - o_ref).max() <= O_TOL
    _check_lse(got["lse"], lse_ref)
    dq, dk, dv = oracle.spa_bwd(qf, kf, vf, dof, scale, lo_o, hi_o)
    _check_grad(got["dq"], dq, "dq")
    _check_grad(got["dk"], dk, "dk")
    _check_grad(got["dv"], dv, "dv")
    return got


SMALL_WORKLOADS = ["b1_h4_n256_d64", "b1_h8_n1024_d64", "b1_h8_n1000_d64", "b1_h8_n1001_d64"]


@pytest.mark.parametrize("name", SMALL_WORKLOADS)
def test_small_workloads_every_element(spa, name):
    w = synth.WORKLOADS[name]
    q, k, v, do = synth.workload_inputs(w)
    _full_check(spa, q, k, v, do, w.scale)


# shapes that span several tiles, ragged tails, width-1 bands, one head,
# both head dims, batches > 1
EDGE_SHAPES = [
    (1, 1, 1, 64), (1, 1, 1, 128), (1, 1, 200, 64), (2, 1, 384, 128), (1, 3, 129, 128),
    (1, 4, 127, 64), (2, 5, 777, 128), (1, 64, 64, 64), (1, 256, 256, 64), (1, 2, 130, 128),
    (3, 7, 500, 64), (1, 8, 2048, 128),
]


@pytest.mark.parametrize("B,H,N,d", EDGE_SHAPES)
def test_edge_shapes_every_element(spa, B, H, N, d):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=7 + N + H)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d))


# Plain bands at d = 128 where the dK/dV and dQ passes run more than one unit
# per CTA (the persistent grid has at most 148 CTAs): unit boundaries, the
# epilogue overlapping the next unit's first steps, TMEM reuse across units.
# B1 H16 N4096: 272 key-tile units, 272 query-tile units; B2 H8 N3000: a
# ragged tail and bands of width 375.
MULTI_UNIT_SHAPES = [(1, 16, 4096, 128), (2, 8, 3000, 128)]


@pytest.mark.parametrize("B,H,N,d", MULTI_UNIT_SHAPES)
def test_multi_unit_per_cta_every_element(spa, B, H, N, d):
    lo, _ = oracle.bands(N, H)
    units = B * sum((N - 1 - int(l)) // 128 + 1 for l in lo)
    assert units > 148  # more units than CTAs on a B200
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=17 + N + H)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d))


# Mean band width of at least 768: the forward's two softmax warpgroups take
# turns (the narrower shapes above run them freely), with ragged tails and both
# head dims; the last two are dense causal attention on every head.
WIDE_SHAPES = [(1, 1, 1000, 64), (2, 2, 1777, 128), (1, 3, 2500, 64), (1, 1, 3001, 128)]


@pytest.mark.parametrize("B,H,N,d", WIDE_SHAPES)
def test_wide_bands_every_element(spa, B, H, N, d):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=11 + N + H)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d))


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 1100, 64), (2, 3, 900, 128)])
def test_full_bands_every_element(spa, B, H, N, d):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=13 + N)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d), [0] * H, [N] * H)


@pytest.mark.parametrize("kind", ["full", "first_half", "shared_window", "odd"])
def test_explicit_bands(spa, kind):
    B, H, N, d = 1, 4, 600, 64
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=99)
    lo, hi = oracle.bands(N, H)
    if kind == "full":           # dense causal attention on every head
        lo, hi = [0] * H, [N] * H
    elif kind == "first_half":   # first half of each band
        hi = [int(a + max((b - a) // 2, 1)) for a, b in zip(lo, hi)]
        lo = [int(a) for a in lo]
    elif kind == "shared_window":  # every head the same local window
        lo, hi = [0] * H, [96] * H
    else:
        lo, hi = [0, 3, 257, 599], [1, 400, 300, 600]
    _full_check(spa, q, k, v, do, 0.125, [int(x) for x in lo], [int(x) for x in hi])


@pytest.mark.parametrize("B,H,N,d", [(1, 8, 1001, 64), (2, 5, 777, 128), (1, 3, 129, 128), (1, 4, 300, 128)])
def test_backward_step_entry_points(spa, B, H, N, d):
    # The three-step entry points (D kernel, dk/dv pass, dq pass) and the
    # fused dq pass that forms D itself, followed by the dk/dv pass, both give
    # the oracle's gradients; the D each leaves in the workspace matches its
    # definition evaluated in fp64 on the same bf16 o and dout.
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=31 + N + d)
    scale = 1 / math.sqrt(d)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = spa.attention_forward(qd, kd, vd, scale)
    rows = B * H * N
    ws3 = torch.full((spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4,), float("nan"), device=dev)
    wsf = torch.full_like(ws3, float("nan"))
    g3 = [torch.empty_like(qd) for _ in range(3)]  # dq, dk, dv
    gf = [torch.empty_like(qd) for _ in range(3)]
    spa.spa_attn_bwd_preprocess(o, dod, ws3)
    spa.spa_attn_bwd_dkdv(qd, kd, vd, dod, lse, ws3, g3[1], g3[2], scale)
    spa.spa_attn_bwd_dq(qd, kd, vd, dod, lse, ws3, g3[0], scale)
    spa.spa_attn_bwd_dq_delta(qd, kd, vd, o, dod, lse, wsf, gf[0], scale)
    spa.spa_attn_bwd_dkdv(qd, kd, vd, dod, lse, wsf, gf[1], gf[2], scale)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK

    d_ref = (o.double() * dod.double()).sum(-1).reshape(-1).cpu().numpy()
    d3 = ws3[:rows].double().cpu().numpy()
    df = wsf[:rows].double().cpu().numpy()
    tol = 1e-5 + 1e-5 * np.abs(d_ref)
    assert (np.abs(d3 - d_ref) <= tol).all()
    # the fused pass writes D for every row of the 128-row query blocks some
    # band reaches: rows from 128 * floor(lo_h / 128) on
    lo, _ = oracle.bands(N, H)
    written = np.zeros((B, H, N), dtype=bool)
    for h in range(H):
        written[:, h, (int(lo[h]) // 128) * 128:] = True
    written = written.reshape(-1)
    assert (np.abs(df[written] - d_ref[written]) <= tol[written]).all()

    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    refs = oracle.spa_bwd(qf, kf, vf, dof, scale)
    for got in (g3, gf):
        for g, ref, name in zip(got, refs, ("dq", "dk", "dv")):
            _check_grad(_f64(g), ref, name)


def test_dense_causal_equals_torch_sdpa_in_fp32(spa):
    # an independent library path: full bands on every head is causal attention
    B, H, N, d = 2, 4, 512, 128
    q, k, v, _ = synth.make_inputs(B, H, N, d, seed=5)
    got = _gpu_run(spa, q, k, v, q, 1 / math.sqrt(d), [0] * H, [N] * H, backward=False)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.float(), k.float(), v.float(), is_causal=True).double().numpy()
    assert np.abs(got["o"] - ref).max() <= O_TOL


def test_deterministic(spa):
    w = synth.WORKLOADS["b1_h8_n1001_d64"]
    q, k, v, do = synth.workload_inputs(w)
    a = _gpu_run(spa, q, k, v, do, w.scale)
    b = _gpu_run(spa, q, k, v, do, w.scale)
    for name in a:
        assert np.array_equal(a[name], b[name], equal_nan=True), name


def test_autograd_function(spa):
    B, H, N, d = 1, 4, 300, 64
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=3)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    o = spa.spattention(qd, kd, vd)
    o.backward(do.to(dev))
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, _ = oracle.spa_fwd(qf, kf, vf, d ** -0.5)
    assert np.abs(_f64(o) - o_ref).max() <= O_TOL
    for g, ref, n in zip((qd.grad, kd.grad, vd.grad), oracle.spa_bwd(qf, kf, vf, dof, d ** -0.5),
                         "qkv"):
        _check_grad(_f64(g), ref, n)


def test_autograd_function_with_the_one_pass_backward(spa):
    B, H, N, d = 2, 4, 700, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=19)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    o = spa.spattention(qd, kd, vd, backward="fused")
    o.backward(do.to(dev))
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    o_ref, _ = oracle.spa_fwd(qf, kf, vf, d ** -0.5)
    assert np.abs(_f64(o) - o_ref).max() <= O_TOL
    for g, ref, n in zip((qd.grad, kd.grad, vd.grad), oracle.spa_bwd(qf, kf, vf, dof, d ** -0.5), "qkv"):
        _check_grad(_f64(g), ref, n)
    with pytest.raises(ValueError):
        spa.spattention(qd, kd, vd, backward="other")


@pytest.mark.parametrize("B,H,N,d,explicit", [(3, 4, 1000, 64, False), (2, 8, 4096, 128, False),
                                             (2, 3, 700, 128, True), (1, 32, 2048, 128, False)])
def test_decode_matches_the_forward_row(spa, B, H, N, d, explicit):
    # One new token per sequence: the result equals the oracle's forward row
    # pos[b] of the sequence whose row pos[b] holds the token's query.
    q, k, v, _ = synth.make_inputs(B, H, N, d, seed=41 + N + d)
    tok = synth.make_inputs(B, H, 1, d, seed=43 + N)[0][:, :, 0, :].contiguous()  # [B, H, d]
    lo, hi = (None, None)
    if explicit:
        lo, hi = [0, 5, 300], [700, 6, 457]
    blo = np.array(oracle.bands(N, H)[0] if lo is None else lo)
    scale = 1 / math.sqrt(d)
    dev = torch.device("cuda:0")
    kd, vd, tokd = k.to(dev), v.to(dev), tok.to(dev)
    rng = np.random.default_rng(N)
    # positions: start, the band edges, the end, random ones
    cands = sorted({0, 1, int(blo.max()) - 1, int(blo.max()), int(blo[1]) if H > 1 else 1, N - 2, N - 1}
                   | set(int(x) for x in rng.integers(0, N, 6)))
    cands = [c for c in cands if 0 <= c < N]
    for start in range(0, len(cands), B):
        pos = np.array([cands[(start + b) % len(cands)] for b in range(B)], dtype=np.int32)
        o, lse = spa.attention_decode(tokd, kd, vd, torch.from_numpy(pos).to(dev), scale, lo, hi)
        torch.cuda.synchronize()
        assert spa.spa_device_status() == spa.SPA_OK
        qfull = q.clone()
        for b in range(B):
            qfull[b, :, pos[b], :] = tok[b]
        rows = [(b * H + h) * N + int(pos[b]) for b in range(B) for h in range(H)]
        o_ref, lse_ref = oracle.spa_fwd_rows(_f64(qfull), _f64(k), _f64(v), scale, rows,
                                             None if lo is None else np.array(lo),
                                             None if hi is None else np.array(hi))
        got_o = _f64(o).reshape(B * H, d)
        assert not np.isnan(got_o).any()
        assert np.abs(got_o - o_ref).max() <= O_TOL
        _check_lse(_f64(lse).reshape(-1), lse_ref)
    # positions outside [0, N): o = 0, lse = -inf
    pos = torch.tensor([N, -1][:B] + [0] * max(0, B - 2), dtype=torch.int32, device=dev)
    o, lse = spa.attention_decode(tokd, kd, vd, pos, scale, lo, hi)
    torch.cuda.synchronize()
    for b in range(min(B, 2)):
        assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))


def test_decode_full_size_sampled_heads(spa):
    # The decode bench's cache shape (H32, N32768, d128), two sequences at
    # different positions; sampled heads are checked against the oracle's
    # forward row on that head's slice of the cache.
    B, H, N, d = 2, 32, 32768, 128
    q, k, v, _ = synth.make_inputs(B, H, N, d, seed=77)
    tok = q[:, :, 0, :].contiguous()
    dev = torch.device("cuda:0")
    pos = np.array([N - 1, 20011], dtype=np.int32)
    scale = 1 / math.sqrt(d)
    o, lse = spa.attention_decode(tok.to(dev), k.to(dev), v.to(dev), torch.from_numpy(pos).to(dev), scale)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    lo, hi = oracle.bands(N, H)
    for b in range(B):
        for h in (0, 1, 13, 30, 31):
            ks, vs = _f64(k[b:b + 1, h:h + 1]), _f64(v[b:b + 1, h:h + 1])
            qs = np.zeros_like(ks)
            qs[0, 0, pos[b]] = _f64(tok[b, h])
            o_ref, lse_ref = oracle.spa_fwd_rows(qs, ks, vs, scale, [int(pos[b])], [int(lo[h])], [int(hi[h])])
            assert np.abs(_f64(o[b, h]) - o_ref[0]).max() <= O_TOL, (b, h)
            _check_lse(_f64(lse[b, h]).reshape(1), lse_ref)


def test_calls_from_a_fresh_thread(spa):
    # a host thread that has made no CUDA call yet (as autograd's worker
    # thread may be) gets the same results as the main thread
    import threading
    B, H, N, d = 1, 4, 300, 64
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=5)
    want = _gpu_run(spa, q, k, v, do, 0.125)
    got, errors = {}, []

    def run():
        try:
            got.update(_gpu_run(spa, q, k, v, do, 0.125))
        except Exception as e:  # reported below, in the test's own thread
            errors.append(e)

    t = threading.Thread(target=run)
    t.start()
    t.join()
    assert not errors, errors
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(got[name], want[name]), name


@pytest.mark.parametrize("N,H,Bq,Bk", [(1024, 8, 128, 128), (1001, 8, 64, 128), (1001, 8, 128, 64),
                                       (4096, 16, 128, 128), (97, 7, 16, 8)])
def test_tile_classes_on_device_bit_exact(spa, N, H, Bq, Bk):
    nqt, nkt = -(-N // Bq), -(-N // Bk)
    out = torch.full((H, nqt, nkt), 255, dtype=torch.uint8, device="cuda:0")
    spa.spa_tile_classes_device(N, H, Bq, Bk, out)
    lo, hi = oracle.bands(N, H)
    np.testing.assert_array_equal(out.cpu().numpy(), oracle.tile_classes(N, lo, hi, Bq, Bk))


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times:
# sampled rows against the oracle's one-row entry points
# ---------------------------------------------------------------------------
LARGE = ["b8_h16_n4096_d128", "b4_h32_n8192_d128", "b1_h32_n32768_d128", "b1_h32_n30001_d128"]


def _targeted_key_rows(B, H, N, lo):
    """Key rows of every head (in batch h mod B) where the dK/dV pass changes
    regime: the last key some query reaches (N - 1 - lo_h), the first that
    none does (N - lo_h, whose dk and dv must be exactly 0), both sides of
    the 128-key tile boundaries at the first tile, the middle of the head
    and the last reached tile, and the last key of the sequence (the ragged
    tail tile when N is not a multiple of 128)."""
    out = []
    for h in range(H):
        last = N - 1 - int(lo[h])
        tiles = {1, (N // 2) // 128, last // 128}
        cand = {last, last + 1, N - 1} | {128 * t - 1 for t in tiles} | {128 * t for t in tiles}
        base = ((h % B) * H + h) * N
        out += [base + j for j in cand if 0 <= j < N]
    return out


def _sampled_check(spa, w, n_random, n_key_rows, full_bands=False, bwd="two-pass"):
    q, k, v, do = synth.workload_inputs(w)
    B, H, N, d = w.B, w.H, w.N, w.d
    if full_bands:  # [0, N) on every head: dense causal attention per head
        lo, hi = np.zeros(H, dtype=np.int64), np.full(H, N, dtype=np.int64)
        got = _gpu_run(spa, q, k, v, do, w.scale, [0] * H, [N] * H, bwd=bwd)
    else:
        lo, hi = oracle.bands(N, H)
        got = _gpu_run(spa, q, k, v, do, w.scale, bwd=bwd)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert not np.isnan(got[name]).any(), name
    per_head = [[int(lo[h]) - 1, int(lo[h]), int(lo[h]) + 1, int(lo[h]) + 127, int(lo[h]) + 128]
                for h in range(H)]
    rows = synth.sample_rows(B, H, N, n_random, seed=w.seed, per_head=per_head)
    g = torch.Generator().manual_seed(w.seed + 1)
    key_rows = sorted(set(torch.randint(0, B * H * N, (n_key_rows,), generator=g).tolist())
                      | set(_targeted_key_rows(B, H, N, lo)))
    flat = lambda x: x.reshape(B * H * N, -1)
    ok = {"o": [], "dq": [], "dk": [], "dv": []}
    refs = {"o": [], "dq": [], "dk": [], "dv": []}
    lse_got, lse_ref = [], []
    # group rows by (b, h) and hand the oracle one head at a time
    for bh in sorted(set(r // N for r in rows) | set(r // N for r in key_rows)):
        h = bh % H
        sl = lambda t: _f64(t.reshape(B * H, N, d)[bh])[None, None]
        qh, kh, vh, doh = sl(q), sl(k), sl(v), sl(do)
        blo, bhi = lo[h:h + 1], hi[h:h + 1]
        rs = [r % N for r in rows if r // N == bh]
        if rs:
            o_r, l_r = oracle.spa_fwd_rows(qh, kh, vh, w.scale, rs, blo, bhi)
            dq_r = oracle.spa_bwd_dq_rows(qh, kh, vh, doh, w.scale, rs, blo, bhi)
            idx = [bh * N + i for i in rs]
            ok["o"].append(flat(got["o"])[idx]); refs["o"].append(o_r)
            ok["dq"].append(flat(got["dq"])[idx]); refs["dq"].append(dq_r)
            lse_got.append(got["lse"].reshape(-1)[idx]); lse_ref.append(l_r)
        ks = [r % N for r in key_rows if r // N == bh]
        if ks:
            dk_r, dv_r = oracle.spa_bwd_dkdv_rows(qh, kh, vh, doh, w.scale, ks, blo, bhi)
            idx = [bh * N + j for j in ks]
            ok["dk"].append(flat(got["dk"])[idx]); refs["dk"].append(dk_r)
            ok["dv"].append(flat(got["dv"])[idx]); refs["dv"].append(dv_r)
    # keys that no query reaches (j > N - 1 - lo_h) get exactly zero
    unreached = [r for r in key_rows if (r % N) > N - 1 - int(lo[(r // N) % H])]
    for name in ("dk", "dv"):
        assert not flat(got[name])[unreached].any(), name
    cat = lambda xs: np.concatenate(xs, axis=0)
    assert np.abs(cat(ok["o"]) - cat(refs["o"])).max() <= O_TOL
    _check_lse(np.concatenate(lse_got), np.concatenate(lse_ref))
    for name in ("dq", "dk", "dv"):
        _check_grad(cat(ok[name]), cat(refs[name]), name)


@pytest.mark.parametrize("name", LARGE)
def test_full_size_workloads_sampled_rows(spa, name):
    w = synth.WORKLOADS[name]
    _sampled_check(spa, w, n_random=48, n_key_rows=12)


def test_full_bands_full_size_sampled_rows(spa):
    # the dense-causal-per-head run the benchmark times beside the bands
    _sampled_check(spa, synth.WORKLOADS["b4_h32_n8192_d128"], n_random=24, n_key_rows=8, full_bands=True)


def test_device_wait_timeout_reports_and_recovers(spa):
    # a wait that nothing completes gives up after its limit: the kernel
    # returns, the status word says so once, and the context keeps working
    assert spa.spa_device_status() == spa.SPA_OK
    spa.spa_debug_wait_timeout(20_000_000)  # 20 ms
    assert spa.spa_device_status() == spa.SPA_ERR_TIMEOUT
    assert spa.spa_device_status() == spa.SPA_OK  # cleared by the read
    w = synth.WORKLOADS["b1_h4_n256_d64"]
    q, k, v, do = synth.workload_inputs(w)
    _full_check(spa, q, k, v, do, w.scale)


# ---------------------------------------------------------------------------
# the one-pass backward (spa_attn_bwd_fused): the same gradients, dq summed
# over key tiles in fp32 by reductions; every element on small shapes, sampled
# rows at full size, the same tolerances
# ---------------------------------------------------------------------------
FUSED_SHAPES = EDGE_SHAPES + MULTI_UNIT_SHAPES + WIDE_SHAPES


@pytest.mark.parametrize("B,H,N,d", FUSED_SHAPES)
def test_fused_backward_every_element(spa, B, H, N, d):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=23 + N + H + d)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d), bwd="fused")


@pytest.mark.parametrize("kind", ["full", "first_half", "odd"])
def test_fused_backward_explicit_bands(spa, kind):
    B, H, N, d = 1, 4, 600, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=101)
    lo, hi = oracle.bands(N, H)
    if kind == "full":
        lo, hi = [0] * H, [N] * H
    elif kind == "first_half":
        hi = [int(a + max((b - a) // 2, 1)) for a, b in zip(lo, hi)]
        lo = [int(a) for a in lo]
    else:
        lo, hi = [0, 3, 257, 599], [1, 400, 300, 600]
    _full_check(spa, q, k, v, do, 0.125, [int(x) for x in lo], [int(x) for x in hi], bwd="fused")


@pytest.mark.parametrize("name", SMALL_WORKLOADS)
def test_fused_backward_small_workloads(spa, name):
    w = synth.WORKLOADS[name]
    q, k, v, do = synth.workload_inputs(w)
    _full_check(spa, q, k, v, do, w.scale, bwd="fused")


@pytest.mark.parametrize("name", LARGE)
def test_fused_backward_full_size_sampled_rows(spa, name):
    _sampled_check(spa, synth.WORKLOADS[name], n_random=32, n_key_rows=8, bwd="fused")


def test_fused_backward_dk_dv_match_the_two_pass_backward(spa):
    # dk and dv come from the same products in the same order as the dK/dV
    # pass; only D is summed in another order (one row sum per thread group
    # instead of inside the dQ pass), so they agree to a few bf16 ulps, and
    # dq agrees within the fp32 reassociation of its sums
    B, H, N, d = 1, 8, 2048, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=5)
    a = _gpu_run(spa, q, k, v, do, 1 / math.sqrt(d))
    b = _gpu_run(spa, q, k, v, do, 1 / math.sqrt(d), bwd="fused")
    for name in ("dq", "dk", "dv"):
        scale = np.abs(a[name]).max()
        assert np.abs(a[name] - b[name]).max() <= 2e-2 * scale, name


# ---------------------------------------------------------------------------
# the backward that stores dS (spa_attn_bwd_stored): the dK/dV pass writes
# every tile pair's dS^T, the dQ pass contracts it with k; every element on
# small shapes, sampled rows at full size, the same tolerances
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,H,N,d", FUSED_SHAPES)
def test_stored_backward_every_element(spa, B, H, N, d):
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=29 + N + H + d)
    _full_check(spa, q, k, v, do, 1 / math.sqrt(d), bwd="stored")


@pytest.mark.parametrize("kind", ["full", "first_half", "odd"])
def test_stored_backward_explicit_bands(spa, kind):
    B, H, N, d = 1, 4, 600, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=103)
    lo, hi = oracle.bands(N, H)
    if kind == "full":
        lo, hi = [0] * H, [N] * H
    elif kind == "first_half":
        hi = [int(a + max((b - a) // 2, 1)) for a, b in zip(lo, hi)]
        lo = [int(a) for a in lo]
    else:
        lo, hi = [0, 3, 257, 599], [1, 400, 300, 600]
    _full_check(spa, q, k, v, do, 0.125, [int(x) for x in lo], [int(x) for x in hi], bwd="stored")


@pytest.mark.parametrize("name", SMALL_WORKLOADS)
def test_stored_backward_small_workloads(spa, name):
    w = synth.WORKLOADS[name]
    q, k, v, do = synth.workload_inputs(w)
    _full_check(spa, q, k, v, do, w.scale, bwd="stored")


@pytest.mark.parametrize("name", LARGE)
def test_stored_backward_full_size_sampled_rows(spa, name):
    _sampled_check(spa, synth.WORKLOADS[name], n_random=32, n_key_rows=8, bwd="stored")


def test_stored_backward_is_bit_reproducible_and_matches_the_two_pass_backward(spa):
    # no reductions in any order: two calls agree bit for bit.  Against the
    # two-pass backward: dk and dv come from the same dK/dV products (only D
    # is summed in another order), dq from the dS^T the dK/dV pass formed
    # (S^T = K Q^T) instead of the dQ pass's own S = Q K^T
    B, H, N, d = 1, 8, 2048, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=7)
    a = _gpu_run(spa, q, k, v, do, 1 / math.sqrt(d), bwd="stored")
    b = _gpu_run(spa, q, k, v, do, 1 / math.sqrt(d), bwd="stored")
    for name in a:
        assert np.array_equal(a[name], b[name]), name
    c = _gpu_run(spa, q, k, v, do, 1 / math.sqrt(d))
    for name in ("dq", "dk", "dv"):
        scale = np.abs(c[name]).max()
        assert np.abs(a[name] - c[name]).max() <= 2e-2 * scale, name


def test_autograd_function_with_the_stored_backward(spa):
    B, H, N, d = 2, 4, 700, 128
    q, k, v, do = synth.make_inputs(B, H, N, d, seed=31)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    o = spa.spattention(qd, kd, vd, backward="stored")
    o.backward(do.to(dev))
    qf, kf, vf, dof = (_f64(t) for t in (q, k, v, do))
    for g, ref, n in zip((qd.grad, kd.grad, vd.grad), oracle.spa_bwd(qf, kf, vf, dof, d ** -0.5), "qkv"):
        _check_grad(_f64(g), ref, n)


def test_stored_backward_step_by_step_equals_the_whole_call(spa):
    # the benchmark times spa_attn_bwd_stored_steps launch by launch (D, then
    # dK/dV storing dS^T, then dQ from the tiles); that composition is the call
    B, H, N, d = 2, 6, 1500, 128
    q, k, v, do = (t.to("cuda") for t in synth.make_inputs(B, H, N, d, seed=37))
    scale = 1 / math.sqrt(d)
    o, lse = spa.attention_forward(q, k, v, scale)
    ws = torch.empty(spa.spa_attn_bwd_stored_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    whole = [torch.empty_like(q) for _ in range(3)]
    spa.spa_attn_bwd_stored(q, k, v, o, do, lse, *whole, ws, scale)
    parts = [torch.empty_like(q) for _ in range(3)]
    ws.fill_(0xFF)  # nothing of the first call may be left for the second
    for st in (1, 2, 4):
        spa.spa_attn_bwd_stored(q, k, v, o, do, lse, *parts, ws, scale, steps=st)
    torch.cuda.synchronize()
    assert spa.spa_device_status() == spa.SPA_OK
    for a, b, n in zip(whole, parts, ("dq", "dk", "dv")):
        assert torch.equal(a, b), n
