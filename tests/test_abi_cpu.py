"""CPU-side checks of the C-ABI library: it loads, exports every symbol that
include/spa.h declares, and its host code (bands, tile schedule, argument
checks) is right.  No compute call reaches a GPU here."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from head_partitioned_distance_b200 import spa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "spa.h")).read()
    return set(re.findall(r"SPA_API\s+[\w\s\*]+?\b(spa_\w+)\s*\(", src))


def test_header_declares_the_abi():
    names = _declared_symbols()
    for must in ("spa_band_bounds", "spa_attn_fwd", "spa_attn_bwd", "spa_attn_fwd_ex",
                 "spa_attn_bwd_ex", "spa_attn_bwd_workspace_bytes", "spa_tile_schedule",
                 "spa_device_status", "spa_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(spa.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    # and the binding marshals exactly those
    assert set(spa.EXPORTS) == _declared_symbols()


def test_status_strings_and_version():
    for s in range(5):
        assert spa.spa_status_string(s).startswith("SPA_")
    assert spa.spa_version() >= 100


def test_band_bounds_bit_exact_against_oracle():
    for N in range(1, 130):
        for H in range(1, N + 1):
            lo, hi = spa.spa_band_bounds(N, H)
            olo, ohi = oracle.bands(N, H)
            assert lo == olo.tolist() and hi == ohi.tolist()
    for N, H in [(4096, 16), (8192, 32), (32768, 32), (30001, 32), (1001, 8), (1000, 8),
                 (2 ** 31 - 1, 256), (2 ** 31 - 1, 7)]:
        lo, hi = spa.spa_band_bounds(N, H)
        olo, ohi = oracle.bands(N, H)
        assert lo == olo.tolist() and hi == ohi.tolist()


def test_band_bounds_rejects_bad_requests():
    for N, H in [(0, 1), (3, 4), (5, 0), (2 ** 31, 2)]:
        with pytest.raises(spa.SpaError) as e:
            spa.spa_band_bounds(N, H)
        assert e.value.status == spa.SPA_ERR_INVAL


# Tile sizes the kernels use: forward (128, 128), dK/dV pass (64 queries x
# 128 keys), dQ pass (128 queries x 64 keys); plus odd sizes.
TILE_CASES = [
    (256, 4, 128, 128), (256, 4, 64, 128), (256, 4, 128, 64),
    (1024, 8, 128, 128), (1000, 8, 128, 128), (1001, 8, 64, 128), (1001, 8, 128, 64),
    (777, 5, 128, 128), (256, 256, 128, 128), (255, 200, 64, 128), (130, 2, 128, 128), (1, 1, 128, 128),
    (129, 3, 128, 128), (97, 7, 16, 8), (4096, 16, 128, 128), (4096, 16, 64, 128),
]


@pytest.mark.parametrize("N,H,Bq,Bk", TILE_CASES)
def test_tile_schedule_bit_exact_against_brute_force(N, H, Bq, Bk):
    sch = spa.spa_tile_schedule(N, H, Bq, Bk)
    lo, hi = oracle.bands(N, H)
    want = oracle.tile_classes(N, lo, hi, Bq, Bk)
    np.testing.assert_array_equal(sch["tile_class"], want)
    nqt, nkt = want.shape[1:]
    for h in range(H):
        for t in range(nqt):
            us = np.nonzero(want[h, t])[0]
            if len(us) == 0:
                assert sch["kt_end"][h, t] < sch["kt_begin"][h, t]
            else:
                # the strip is exactly the contiguous run of non-empty tiles
                assert (sch["kt_begin"][h, t], sch["kt_end"][h, t]) == (us[0], us[-1])
                assert len(us) == us[-1] - us[0] + 1
        for u in range(nkt):
            ts = np.nonzero(want[h, :, u])[0]
            if len(ts) == 0:
                assert sch["qt_end"][h, u] < sch["qt_begin"][h, u]
            else:
                assert (sch["qt_begin"][h, u], sch["qt_end"][h, u]) == (ts[0], ts[-1])
                assert len(ts) == ts[-1] - ts[0] + 1


@pytest.mark.parametrize("N,H,h_list", [(8192, 32, [0, 1, 15, 31]), (30001, 32, [0, 7, 31]),
                                        (32768, 32, [0, 31])])
def test_tile_schedule_large_heads_against_brute_force(N, H, h_list):
    # brute force over whole tiles is quadratic in N; check selected heads
    lo, hi = oracle.bands(N, H)
    sch = spa.spa_tile_schedule(N, H, 128, 128)
    for h in h_list:
        want = oracle.tile_classes(N, lo[h:h + 1], hi[h:h + 1], 128, 128)
        np.testing.assert_array_equal(sch["tile_class"][h], want[0])


def test_tile_schedule_explicit_bands():
    N = 500
    lo = [0, 0, 37, 100, 499]
    hi = [500, 1, 250, 101, 500]
    sch = spa.spa_tile_schedule(N, 5, 128, 64, lo, hi)
    want = oracle.tile_classes(N, lo, hi, 128, 64)
    np.testing.assert_array_equal(sch["tile_class"], want)


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_entry_points_reject_bad_arguments_before_any_launch():
    L = spa._lib
    p = _fake(1 << 20)  # never dereferenced: every call below fails its checks first
    f = lambda *a: L.spa_attn_fwd(p, p, p, p, p, *a, None)
    assert f(1, 4, 256, 96, 0.1) == spa.SPA_ERR_UNSUPPORTED      # d
    assert f(1, 300, 400, 64, 0.1) == spa.SPA_ERR_UNSUPPORTED    # H > 256
    assert f(1, 8, 4, 64, 0.1) == spa.SPA_ERR_INVAL              # H > N
    assert f(0, 4, 256, 64, 0.1) == spa.SPA_ERR_INVAL            # B
    assert f(1, 4, 0, 64, 0.1) == spa.SPA_ERR_INVAL              # N
    assert f(1, 4, 2 ** 31, 64, 0.1) == spa.SPA_ERR_INVAL        # N too large
    assert f(1, 4, 256, 64, float("nan")) == spa.SPA_ERR_INVAL   # scale
    assert f(1, 4, 256, 64, -0.125) == spa.SPA_ERR_INVAL         # scale must be > 0
    assert f(1, 4, 256, 64, 0.0) == spa.SPA_ERR_INVAL
    assert L.spa_attn_fwd(p, None, p, p, p, 1, 4, 256, 64, 0.1, None) == spa.SPA_ERR_INVAL
    odd = _fake((1 << 20) + 8)
    assert L.spa_attn_fwd(p, p, odd, p, p, 1, 4, 256, 64, 0.1, None) == spa.SPA_ERR_UNSUPPORTED
    # explicit bands: empty, reversed, out of range
    for lo, hi in (([0, 5], [0, 6]), ([3, 1], [2, 9]), ([0, 0], [8, 300])):
        a = (ctypes.c_int32 * 2)(*lo)
        b = (ctypes.c_int32 * 2)(*hi)
        assert L.spa_attn_fwd_ex(p, p, p, p, p, 1, 2, 256, 64, 0.1, a, b, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_fwd_ex(p, p, p, p, p, 1, 2, 256, 64, 0.1, None, None, None) == spa.SPA_ERR_INVAL
    # outputs written in 32-byte stores: 16-byte aligned is not enough
    half = _fake((1 << 20) + 16)
    assert L.spa_attn_fwd(p, p, p, half, p, 1, 4, 256, 64, 0.1, None) == spa.SPA_ERR_UNSUPPORTED
    for pos in (6, 7, 8):  # dq, dk, dv of spa_attn_bwd
        args = [p] * 10
        args[pos] = half
        assert L.spa_attn_bwd(*args, 1, 4, 256, 64, 0.1, None) == spa.SPA_ERR_UNSUPPORTED
    g = lambda *a: L.spa_attn_bwd(p, p, p, p, p, p, p, p, p, p, *a, None)
    assert g(1, 4, 256, 80, 0.1) == spa.SPA_ERR_UNSUPPORTED
    assert g(1, 8, 4, 64, 0.1) == spa.SPA_ERR_INVAL
    assert L.spa_attn_bwd(p, p, p, p, p, p, p, p, p, None, 1, 4, 256, 64, 0.1, None) == spa.SPA_ERR_INVAL


def test_fused_backward_rejects_bad_arguments_before_any_launch():
    L = spa._lib
    p = _fake(1 << 20)
    f = lambda *a, steps=7: L.spa_attn_bwd_fused_steps(*a, 1, 4, 256, 64, 0.1, None, None, None, steps)
    ten = [p] * 10
    assert f(*ten, steps=0) == spa.SPA_ERR_INVAL
    assert f(*ten, steps=8) == spa.SPA_ERR_INVAL
    for i in range(10):  # every pointer is required
        args = list(ten)
        args[i] = None
        assert f(*args) == spa.SPA_ERR_INVAL
        assert L.spa_attn_bwd_fused(*args, 1, 4, 256, 64, 0.1, None, None, None) == spa.SPA_ERR_INVAL
    half = _fake((1 << 20) + 16)
    for i in (7, 8):  # dk, dv leave in 32-byte stores
        args = list(ten)
        args[i] = half
        assert f(*args) == spa.SPA_ERR_UNSUPPORTED
    args = list(ten)
    args[9] = _fake((1 << 20) + 128)  # workspace must be 256-byte aligned
    assert f(*args) == spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_bwd_fused(*ten, 1, 4, 256, 96, 0.1, None, None, None) == spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_bwd_fused(*ten, 1, 8, 4, 64, 0.1, None, None, None) == spa.SPA_ERR_INVAL


def test_stored_backward_rejects_bad_arguments_before_any_launch():
    L = spa._lib
    p = _fake(1 << 20)
    f = lambda *a, B=1, H=4, N=256, d=64: L.spa_attn_bwd_stored(*a, B, H, N, d, 0.1, None, None, None)
    ten = [p] * 10
    for i in range(10):  # every pointer is required
        args = list(ten)
        args[i] = None
        assert f(*args) == spa.SPA_ERR_INVAL
    half = _fake((1 << 20) + 16)
    for i in (6, 7, 8):  # dq, dk, dv leave in 32-byte stores
        args = list(ten)
        args[i] = half
        assert f(*args) == spa.SPA_ERR_UNSUPPORTED
    args = list(ten)
    args[9] = _fake((1 << 20) + 128)  # workspace must be 256-byte aligned
    assert f(*args) == spa.SPA_ERR_UNSUPPORTED
    assert f(*ten, d=96) == spa.SPA_ERR_UNSUPPORTED
    assert f(*ten, H=8, N=4) == spa.SPA_ERR_INVAL
    # more dS^T tiles than a 32-bit index holds
    assert f(*ten, B=65535, H=256, N=2 ** 20) == spa.SPA_ERR_UNSUPPORTED
    assert spa.spa_attn_bwd_stored_workspace_bytes(65535, 256, 2 ** 20, 64) == 0
    st = lambda steps: L.spa_attn_bwd_stored_steps(*ten, 1, 4, 256, 64, 0.1, None, None, None, steps)
    assert st(0) == spa.SPA_ERR_INVAL and st(8) == spa.SPA_ERR_INVAL


@pytest.mark.parametrize("N,H,lo,hi", [(32768, 32, None, None), (30001, 32, None, None), (8192, 32, None, None),
                                       (1001, 8, None, None), (129, 3, None, None),
                                       (500, 5, [0, 0, 37, 100, 499], [500, 1, 250, 101, 500])])
def test_stored_workspace_holds_every_tile_pair(N, H, lo, hi):
    # D, padded to 1024 bytes, then the dS^T tiles (128 x 128 bf16): head h
    # owns, per batch and per key tile some query reaches, L_h tiles, where
    # L_h = (hi + 126) // 128 - lo // 128 + 1 must cover the dK/dV strip of
    # every such key tile (the schedule's qt_begin..qt_end, itself checked
    # against the oracle's brute-force tile classes above).  A Balanced
    # Distance Partitioning band that ends well before N reaches the bound; a
    # band that N clips may need a tile less.
    B, d = 2, 128
    got = spa.spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo, hi)
    sch = spa.spa_tile_schedule(N, H, 128, 128, lo, hi)
    if lo is None:
        lo, hi = oracle.bands(N, H)
    tiles = 0
    for h in range(H):
        reached = (N - 1 - int(lo[h])) // 128 + 1
        L = (int(hi[h]) + 126) // 128 - int(lo[h]) // 128 + 1
        strips = sch["qt_end"][h] - sch["qt_begin"][h] + 1
        assert (strips[:reached] >= 1).all() and (strips[reached:] <= 0).all()
        assert strips.max() <= L
        tiles += B * reached * L
    if N in (32768, 30001, 8192):
        assert all((hh + 126) // 128 - ll // 128 + 1 == (sch["qt_end"][h] - sch["qt_begin"][h] + 1).max()
                   for h, (ll, hh) in enumerate(zip(lo, hi)) if hh <= N - 256)
    assert got == -(-4 * B * H * N // 1024) * 1024 + tiles * 32768


def test_fused_workspace_size():
    # D (fp32 per row, padded to 256 bytes), then the fp32 dq sums
    assert spa.spa_attn_bwd_fused_workspace_bytes(1, 32, 32768, 128) == 4 * 32 * 32768 * (1 + 128)
    assert spa.spa_attn_bwd_fused_workspace_bytes(1, 1, 3, 64) == 256 + 4 * 3 * 64
    assert spa.spa_attn_bwd_fused_workspace_bytes(1, 1, 3, 96) == 0


def test_workspace_size():
    assert spa.spa_attn_bwd_workspace_bytes(4, 32, 8192) == 4 * 32 * 8192 * 4
    assert spa.spa_attn_bwd_workspace_bytes(0, 1, 1) == 0


def test_decode_rejects_bad_arguments_and_sizes_its_workspace():
    L = spa._lib
    p = _fake(1 << 20)  # never dereferenced: every call below fails its checks first
    f = lambda *a: L.spa_attn_decode(p, p, p, p, p, p, p, *a, None, None, None)
    assert f(1, 4, 256, 96, 0.1) == spa.SPA_ERR_UNSUPPORTED      # d
    assert f(1, 300, 400, 64, 0.1) == spa.SPA_ERR_UNSUPPORTED    # H > 256
    assert f(1, 8, 4, 64, 0.1) == spa.SPA_ERR_INVAL              # H > N
    assert f(1, 4, 256, 64, float("inf")) == spa.SPA_ERR_INVAL   # scale
    assert f(1, 4, 256, 64, 0.0) == spa.SPA_ERR_INVAL
    assert L.spa_attn_decode(p, p, p, None, p, p, p, 1, 4, 256, 64, 0.1, None, None, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_decode(p, p, p, p, p, p, None, 1, 4, 256, 64, 0.1, None, None, None) == spa.SPA_ERR_INVAL
    odd = _fake((1 << 20) + 2)
    assert L.spa_attn_decode(p, p, p, odd, p, p, p, 1, 4, 256, 64, 0.1, None, None, None) == spa.SPA_ERR_UNSUPPORTED
    a, b = (ctypes.c_int32 * 2)(3, 1), (ctypes.c_int32 * 2)(2, 9)     # reversed band
    assert L.spa_attn_decode(p, p, p, p, p, p, p, 1, 2, 256, 64, 0.1, a, b, None) == spa.SPA_ERR_INVAL
    # workspace: one (o[d], m, l) partial per 256-key chunk of the widest band
    assert spa.spa_attn_decode_workspace_bytes(2, 4, 4096, 128) == 2 * 4 * 4 * 130 * 4
    assert spa.spa_attn_decode_workspace_bytes(1, 8, 1001, 64) == 8 * 1 * 66 * 4
    assert spa.spa_attn_decode_workspace_bytes(1, 2, 700, 128, [0, 5], [600, 6]) == 2 * 3 * 130 * 4
    assert spa.spa_attn_decode_workspace_bytes(1, 4, 256, 96) == 0
    assert spa.spa_attn_decode_workspace_bytes(1, 2, 700, 128, [3, 1], [2, 9]) == 0


def test_timeout_hook_rejects_bad_limits():
    L = spa._lib
    assert L.spa_debug_wait_timeout(0, None) == spa.SPA_ERR_INVAL
    assert L.spa_debug_wait_timeout(2_000_000_000, None) == spa.SPA_ERR_INVAL


def test_union_entry_points_reject_bad_arguments_before_any_launch():
    L = spa._lib
    p = _fake(1 << 20)  # never dereferenced: every call below fails its checks first
    B, H, N, d = 1, 4, 256, 64
    args = (B, H, N, d, 0.1)

    def fwd(ws, w, lo=None, hi=None, shape=args):
        # the forward takes no workspace
        return L.spa_attn_fwd_union(p, p, p, p, p, *shape, w, lo, hi, None)

    def bwd(ws, w, lo=None, hi=None, shape=args):
        return L.spa_attn_bwd_union(p, p, p, p, p, p, p, p, p, ws, *shape, w, lo, hi, None)

    assert bwd(None, 8) == spa.SPA_ERR_INVAL                                # workspace
    assert bwd(_fake((1 << 20) + 16), 8) == spa.SPA_ERR_UNSUPPORTED         # 32-byte aligned
    for call in (fwd, bwd):
        assert call(p, 0) == spa.SPA_ERR_INVAL            # window must be >= 1
        assert call(p, N + 1) == spa.SPA_ERR_INVAL        # and <= N
        assert call(p, 8, shape=(B, H, N, 96, 0.1)) == spa.SPA_ERR_UNSUPPORTED
        bad_lo = (ctypes.c_int32 * H)(0, 9, 5, 7)
        bad_hi = (ctypes.c_int32 * H)(4, 3, 6, 300)     # reversed and out-of-range bands
        assert call(p, 8, bad_lo, bad_hi) == spa.SPA_ERR_INVAL
        # H = N with window 1: head 0's set is the single distance 0
        assert call(p, 1, shape=(1, 16, 16, 64, 0.1)) == spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_bwd_union(p, p, p, p, p, p, None, p, p, p, *args, 8, None, None, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_union_merge(p, p, None, p, *args[:4], None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_union_merge(p, p, _fake((1 << 20) + 8), p, *args[:4], None) == spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_union_merge(p, p, p, p, 1, 4, 256, 96, None) == spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_union_add_grads(p, p, p, p, None, p, *args[:4], None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_union_add_grads(p, p, p, p, p, _fake((1 << 20) + 4), *args[:4], None) == \
        spa.SPA_ERR_UNSUPPORTED
    assert L.spa_attn_union_workspace_bytes(1, 4, 256, 96) == 0
    rows = 1 * 4 * 256
    assert L.spa_attn_union_workspace_bytes(1, 4, 256, 64) == rows * 4
    assert L.spa_attn_fwd_merge(p, p, p, None, p, *args, None, None, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_fwd_merge(p, p, p, _fake((1 << 20) + 16), p, *args, None, None, None) == \
        spa.SPA_ERR_UNSUPPORTED
    # the adding backward passes check like the overwriting ones
    assert L.spa_attn_bwd_dkdv_add(p, p, p, p, p, p, None, p, *args, None, None, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_bwd_dq_add(p, p, p, p, p, p, None, *args, None, None, None) == spa.SPA_ERR_INVAL
    assert L.spa_attn_bwd_dq_add(p, p, p, p, p, p, _fake((1 << 20) + 16), *args, None, None, None) == \
        spa.SPA_ERR_UNSUPPORTED


@pytest.mark.parametrize("N,H,w", [(600, 4, 100), (600, 4, 200), (600, 4, 600), (777, 5, 37), (32768, 32, 256),
                                   (16, 16, 2), (1001, 8, 1)])
def test_union_parts_split_each_head_into_two_disjoint_intervals(N, H, w):
    a1, b1, a2, b2 = spa.spa_union_parts(N, H, w)
    lo, hi = oracle.bands(N, H)
    for h in range(H):
        want = set(range(0, w)) | set(range(int(lo[h]), int(hi[h])))
        p1, p2 = set(range(a1[h], b1[h])), set(range(a2[h], b2[h]))
        assert p1 and p2 and not (p1 & p2)
        assert p1 | p2 == want
    with pytest.raises(spa.SpaError):
        spa.spa_union_parts(16, 16, 1)  # head 0 is the single distance 0


def test_step_wrappers_reject_bad_tensors_before_the_library():
    # Every backward step wrapper, like spa_attn_bwd, checks shape, dtype,
    # contiguity, device and the workspace size before it hands pointers to
    # the library; on this CPU-only machine a check that passed would reach
    # the library with host pointers, so each case must raise ValueError.
    from head_partitioned_distance_b200 import spa
    B, H, N, d = 1, 2, 64, 64
    t = lambda *shape, dt=torch.bfloat16: torch.zeros(shape, dtype=dt)
    q, k, v, o, do, dq, dk, dv = (t(B, H, N, d) for _ in range(8))
    lse = t(B, H, N, dt=torch.float32)
    ws = t(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dt=torch.float32)
    short = t(B * H * N // 2, dt=torch.float32)
    bad_do = t(B, H, N - 1, d)
    bad_lse = t(B, H, N, dt=torch.float16)
    calls = [
        lambda: spa.spa_attn_bwd_preprocess(o, do, ws),
        lambda: spa.spa_attn_bwd_preprocess(o, bad_do, ws),
        lambda: spa.spa_attn_bwd_dkdv(q, k, v, do, lse, ws, dk, dv, 0.1),
        lambda: spa.spa_attn_bwd_dkdv(q, k, v, bad_do, lse, ws, dk, dv, 0.1),
        lambda: spa.spa_attn_bwd_dq(q, k, v, do, bad_lse, ws, dq, 0.1),
        lambda: spa.spa_attn_bwd_dkdv_add(q, k, v, do, lse, short, dk, dv, 0.1),
        lambda: spa.spa_attn_bwd_dq_add(q, k, v, do, lse, ws, dq.float(), 0.1),
        lambda: spa.spa_attn_bwd_dq_delta(q, k, v, o, do, lse, ws, dq, 0.1),
        lambda: spa.spa_attn_bwd_dq_delta(q, k, v, o.transpose(2, 3), do, lse, ws, dq, 0.1),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError):
            call()
            pytest.fail(f"call {i} was not rejected")
