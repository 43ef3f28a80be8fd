"""fp64 CPU oracle for SPAttention band-sparse attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this module.  The product path (the CUDA
library in ``head_partitioned_distance_b200`` and its binding) never imports
it, and this module imports nothing from there.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one permitted
set enumerated per row); this file only compiles it with gcc and marshals
numpy arrays.  What each function computes, and which passage of the pages it
follows, is written at the top of ``oracle.c``:

* ``bands``            -- Balanced Distance Partitioning ("Making Every Head
  Count", Figure 1 caption), lo_h = floor(h N / H), hi_h = floor((h+1) N / H).
* ``masked_attn_fwd``/``masked_attn_bwd`` -- softmax over a permitted set
  ("Story of Attention -- Part 4", section 1, Sparse-Attention equation).
* ``spa_fwd``/``spa_bwd`` and their ``_rows`` forms -- the same with
  S_i^h = {j : lo_h <= i - j < hi_h, j <= i}; empty rows give o = 0,
  lse = -inf; gradients derived by hand (the pages give none).
* ``tile_classes``     -- brute-force per-element classification of tiles.
* ``union_fwd``/``union_bwd`` (and ``union_fwd_rows``) -- each head's band
  plus a local window [0, w) shared by every head, S_i^h = {j <= i :
  i - j < w or lo_h <= i - j < hi_h}: a reading of the local sharing that
  the EBALL ablation of "Making Every Head Count" (Figure 2(b)) takes out
  (the pages do not define it).

Parity status: every function is pinned by ``tests/test_oracle_pins.py``
(worked example of the blog post, band invariants, reduction to dense causal
attention via ``torch.nn.functional.scaled_dot_product_attention`` in fp64,
central finite differences, torch autograd, and a hand-worked tile-class
table under ``tests/golden``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_d = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_bands.argtypes = [_i64, _i64, _i64p, _i64p]
        lib.oracle_bands.restype = ctypes.c_int
        lib.oracle_band_pairs.argtypes = [_i64, _i64, _i64]
        lib.oracle_band_pairs.restype = ctypes.c_int64
        lib.oracle_masked_attn_fwd.argtypes = [_d, _d, _d, _u8p, _i64, _i64, _i64,
                                               ctypes.c_double, _d, _d, _d, _d]
        lib.oracle_masked_attn_bwd.argtypes = [_d, _d, _d, _u8p, _i64, _i64, _i64,
                                               ctypes.c_double, _d, _d, _d, _d]
        lib.oracle_spa_fwd.argtypes = [_d, _d, _d, _i64, _i64, _i64, _i64,
                                       ctypes.c_double, _i64p, _i64p, _d, _d]
        lib.oracle_spa_fwd_rows.argtypes = [_d, _d, _d, _i64, _i64, _i64, _i64,
                                            ctypes.c_double, _i64p, _i64p, _i64p, _i64,
                                            _d, _d]
        lib.oracle_spa_bwd.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64,
                                       ctypes.c_double, _i64p, _i64p, _d, _d, _d]
        lib.oracle_spa_bwd_dq_rows.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64,
                                               ctypes.c_double, _i64p, _i64p, _i64p,
                                               _i64, _d]
        lib.oracle_spa_bwd_dkdv_rows.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64,
                                                 ctypes.c_double, _i64p, _i64p, _i64p,
                                                 _i64, _d, _d]
        lib.oracle_tile_classes.argtypes = [_i64, _i64, _i64p, _i64p, _i64, _i64, _u8p]
        lib.oracle_union_fwd.argtypes = [_d, _d, _d, _i64, _i64, _i64, _i64, ctypes.c_double, _i64,
                                         _i64p, _i64p, _d, _d]
        lib.oracle_union_fwd_rows.argtypes = [_d, _d, _d, _i64, _i64, _i64, _i64, ctypes.c_double,
                                              _i64, _i64p, _i64p, _i64p, _i64, _d, _d]
        lib.oracle_union_bwd.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64, ctypes.c_double,
                                         _i64, _i64p, _i64p, _d, _d, _d]
        lib.oracle_union_bwd_dq_rows.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64, ctypes.c_double,
                                                 _i64, _i64p, _i64p, _i64p, _i64, _d]
        lib.oracle_union_bwd_dkdv_rows.argtypes = [_d, _d, _d, _d, _i64, _i64, _i64, _i64,
                                                   ctypes.c_double, _i64, _i64p, _i64p, _i64p, _i64, _d, _d]
        _lib = lib
        return lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64arr(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _pd(a: np.ndarray):
    return a.ctypes.data_as(_d)


def _pi(a: np.ndarray):
    return a.ctypes.data_as(_i64p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def bands(N: int, H: int):
    """Return (lo, hi) int64 arrays of length H."""
    lo = np.zeros(H, np.int64)
    hi = np.zeros(H, np.int64)
    if _load().oracle_bands(N, H, _pi(lo), _pi(hi)) != 0:
        raise ValueError(f"invalid band request N={N} H={H}")
    return lo, hi


def band_pairs(N: int, lo: int, hi: int) -> int:
    """Permitted (i, j) pairs of one head, counted one by one."""
    return int(_load().oracle_band_pairs(N, lo, hi))


def masked_attn_fwd(q, k, v, mask, scale: float):
    """Generic masked attention on one head: q [nq,d], k/v [nk,d], mask [nq,nk].

    Returns (scores, attn, o, lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    nq, d = q.shape
    nk = k.shape[0]
    scores = np.zeros((nq, nk))
    attn = np.zeros((nq, nk))
    o = np.zeros((nq, d))
    lse = np.zeros(nq)
    _load().oracle_masked_attn_fwd(_pd(q), _pd(k), _pd(v), mask.ctypes.data_as(_u8p),
                                   nq, nk, d, scale, _pd(scores), _pd(attn), _pd(o), _pd(lse))
    return scores, attn, o, lse


def masked_attn_bwd(q, k, v, mask, scale: float, dout):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    nq, d = q.shape
    nk = k.shape[0]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    _load().oracle_masked_attn_bwd(_pd(q), _pd(k), _pd(v), mask.ctypes.data_as(_u8p),
                                   nq, nk, d, scale, _pd(dout), _pd(dq), _pd(dk), _pd(dv))
    return dq, dk, dv


def _bands_arg(N, H, lo, hi):
    if lo is None:
        lo, hi = bands(N, H)
    return _i64arr(lo), _i64arr(hi)


def spa_fwd(q, k, v, scale: float, lo=None, hi=None):
    """q, k, v: [B,H,N,d] arrays.  Returns (o [B,H,N,d], lse [B,H,N])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    _load().oracle_spa_fwd(_pd(q), _pd(k), _pd(v), B, H, N, d, scale, _pi(lo), _pi(hi),
                           _pd(o), _pd(lse))
    return o, lse


def spa_fwd_rows(q, k, v, scale: float, rows, lo=None, hi=None):
    """Forward of selected flat rows (b*H + h)*N + i.  Returns (o [n,d], lse [n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    o = np.zeros((len(rows), d))
    lse = np.zeros(len(rows))
    _load().oracle_spa_fwd_rows(_pd(q), _pd(k), _pd(v), B, H, N, d, scale, _pi(lo), _pi(hi),
                                _pi(rows), len(rows), _pd(o), _pd(lse))
    return o, lse


def spa_bwd(q, k, v, dout, scale: float, lo=None, hi=None):
    """Gradients of sum(O * dout).  Returns (dq, dk, dv), each [B,H,N,d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    dq = np.zeros_like(q)
    dk = np.zeros_like(q)
    dv = np.zeros_like(q)
    _load().oracle_spa_bwd(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale,
                           _pi(lo), _pi(hi), _pd(dq), _pd(dk), _pd(dv))
    return dq, dk, dv


def spa_bwd_dq_rows(q, k, v, dout, scale: float, rows, lo=None, hi=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    dq = np.zeros((len(rows), d))
    _load().oracle_spa_bwd_dq_rows(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale,
                                   _pi(lo), _pi(hi), _pi(rows), len(rows), _pd(dq))
    return dq


def spa_bwd_dkdv_rows(q, k, v, dout, scale: float, rows, lo=None, hi=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    dk = np.zeros((len(rows), d))
    dv = np.zeros((len(rows), d))
    _load().oracle_spa_bwd_dkdv_rows(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale,
                                     _pi(lo), _pi(hi), _pi(rows), len(rows), _pd(dk), _pd(dv))
    return dk, dv


def tile_classes(N: int, lo, hi, Bq: int, Bk: int) -> np.ndarray:
    """Brute-force tile classes, uint8 [H, ceil(N/Bq), ceil(N/Bk)]: 0 none, 1 some, 2 all."""
    lo, hi = _i64arr(lo), _i64arr(hi)
    H = len(lo)
    nqt, nkt = -(-N // Bq), -(-N // Bk)
    cls = np.zeros((H, nqt, nkt), np.uint8)
    _load().oracle_tile_classes(N, H, _pi(lo), _pi(hi), Bq, Bk, cls.ctypes.data_as(_u8p))
    return cls


def union_fwd(q, k, v, scale: float, window: int, lo=None, hi=None):
    """Band plus shared local window [0, window).  Returns (o, lse) like spa_fwd."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    _load().oracle_union_fwd(_pd(q), _pd(k), _pd(v), B, H, N, d, scale, int(window), _pi(lo), _pi(hi),
                             _pd(o), _pd(lse))
    return o, lse


def union_fwd_rows(q, k, v, scale: float, window: int, rows, lo=None, hi=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    o = np.zeros((len(rows), d))
    lse = np.zeros(len(rows))
    _load().oracle_union_fwd_rows(_pd(q), _pd(k), _pd(v), B, H, N, d, scale, int(window), _pi(lo),
                                  _pi(hi), _pi(rows), len(rows), _pd(o), _pd(lse))
    return o, lse


def union_bwd(q, k, v, dout, scale: float, window: int, lo=None, hi=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    dq = np.zeros_like(q)
    dk = np.zeros_like(q)
    dv = np.zeros_like(q)
    _load().oracle_union_bwd(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale, int(window),
                             _pi(lo), _pi(hi), _pd(dq), _pd(dk), _pd(dv))
    return dq, dk, dv


def union_bwd_dq_rows(q, k, v, dout, scale: float, window: int, rows, lo=None, hi=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    dq = np.zeros((len(rows), d))
    _load().oracle_union_bwd_dq_rows(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale, int(window),
                                     _pi(lo), _pi(hi), _pi(rows), len(rows), _pd(dq))
    return dq


def union_bwd_dkdv_rows(q, k, v, dout, scale: float, window: int, rows, lo=None, hi=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    lo, hi = _bands_arg(N, H, lo, hi)
    rows = _i64arr(rows)
    dk = np.zeros((len(rows), d))
    dv = np.zeros((len(rows), d))
    _load().oracle_union_bwd_dkdv_rows(_pd(q), _pd(k), _pd(v), _pd(dout), B, H, N, d, scale, int(window),
                                       _pi(lo), _pi(hi), _pi(rows), len(rows), _pd(dk), _pd(dv))
    return dk, dv
