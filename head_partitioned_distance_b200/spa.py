"""Python binding of libspa.so -- argument marshalling only.

Every function here has the name of the C entry point it calls (see
``include/spa.h``) and does nothing but turn torch tensors into pointers and
sizes and the status code into an exception.  All arithmetic runs in the
library's CUDA kernels; there is no fallback of any kind: importing this
module fails when ``libspa.so`` has not been built, and a call fails when the
library reports an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m head_partitioned_distance_b200.build` "
        "(nvcc, sm_100a).  There is no non-CUDA fallback.")

_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float

EXPORTS = {
    "spa_status_string": ([_int], ctypes.c_char_p),
    "spa_version": ([], _int),
    "spa_band_bounds": ([_i64, _int, _i32p, _i32p], _int),
    "spa_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _int, _f32, _vp], _int),
    "spa_attn_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _int, _f32, _i32p, _i32p, _vp],
                        _int),
    "spa_attn_fwd_merge": ([_vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_workspace_bytes": ([_int, _int, _i64], ctypes.c_size_t),
    "spa_attn_bwd": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _vp], _int),
    "spa_attn_bwd_ex": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_preprocess": ([_vp, _vp, _vp, _int, _int, _i64, _int, _vp], _int),
    "spa_attn_bwd_dkdv": ([_vp] * 8 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_dq": ([_vp] * 7 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_dq_delta": ([_vp] * 8 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_dkdv_add": ([_vp] * 8 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_dq_add": ([_vp] * 7 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_decode_workspace_bytes": ([_int, _int, _i64, _int, _i32p, _i32p], ctypes.c_size_t),
    "spa_attn_decode": ([_vp] * 7 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_noalloc": ([_vp] * 9 + [_int, _int, _i64, _int, _f32, _vp], _int),
    "spa_attn_bwd_fused_workspace_bytes": ([_int, _int, _i64, _int], ctypes.c_size_t),
    "spa_attn_bwd_stored_workspace_bytes": ([_int, _int, _i64, _int, _i32p, _i32p], ctypes.c_size_t),
    "spa_attn_bwd_stored": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_stored_steps": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp, _int], _int),
    "spa_attn_bwd_fused": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_fused_steps": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i32p, _i32p, _vp, _int], _int),
    "spa_attn_union_workspace_bytes": ([_int, _int, _i64, _int], ctypes.c_size_t),
    "spa_union_parts": ([_i64, _int, _i64, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p], _int),
    "spa_attn_union_merge": ([_vp] * 4 + [_int, _int, _i64, _int, _vp], _int),
    "spa_attn_union_add_grads": ([_vp] * 6 + [_int, _int, _i64, _int, _vp], _int),
    "spa_attn_fwd_union": ([_vp] * 5 + [_int, _int, _i64, _int, _f32, _i64, _i32p, _i32p, _vp], _int),
    "spa_attn_bwd_union": ([_vp] * 10 + [_int, _int, _i64, _int, _f32, _i64, _i32p, _i32p, _vp], _int),
    "spa_tile_schedule": ([_i64, _int, _i32p, _i32p, _int, _int, _i32p, _i32p, _u8p, _i32p, _i32p],
                          _int),
    "spa_tile_classes_device": ([_i64, _int, _i32p, _i32p, _int, _int, _vp, _vp], _int),
    "spa_debug_wait_timeout": ([_i64, _vp], _int),
    "spa_device_status": ([_vp], _int),
}
for _name, (_args, _res) in EXPORTS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

SPA_OK, SPA_ERR_INVAL, SPA_ERR_UNSUPPORTED, SPA_ERR_CUDA, SPA_ERR_TIMEOUT = 0, 1, 2, 3, 4


class SpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {spa_status_string(status)}")


def _check(status: int, where: str):
    if status != SPA_OK:
        raise SpaError(status, where)


def spa_status_string(status: int) -> str:
    return _lib.spa_status_string(status).decode()


def spa_version() -> int:
    return int(_lib.spa_version())


def _i32(arr):
    a = (ctypes.c_int32 * len(arr))(*[int(x) for x in arr])
    return a


def spa_band_bounds(N: int, H: int):
    """Balanced Distance Partitioning bands: (lo, hi) lists of H ints."""
    lo = (ctypes.c_int32 * H)()
    hi = (ctypes.c_int32 * H)()
    _check(_lib.spa_band_bounds(N, H, lo, hi), "spa_band_bounds")
    return list(lo), list(hi)


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _dims(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("tensors are [B, H, N, d]")
    B, H, N, d = q.shape
    return B, H, N, d


def _need(t: torch.Tensor, shape, dtype, name):
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def spa_attn_fwd(q, k, v, o, lse, scale: float, lo=None, hi=None, stream=None):
    """o, lse = band-sparse attention forward (writes into o [B,H,N,d] bf16 and
    lse [B,H,N] fp32).  lo/hi: optional explicit bands (calls spa_attn_fwd_ex)."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    s = _stream_ptr(stream)
    if lo is None:
        st = _lib.spa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               B, H, N, d, scale, s)
        _check(st, "spa_attn_fwd")
    else:
        st = _lib.spa_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), B, H, N, d, scale, _i32(lo), _i32(hi), s)
        _check(st, "spa_attn_fwd_ex")
    return o, lse


def spa_attn_fwd_merge(q, k, v, o, lse, scale: float, lo=None, hi=None, stream=None):
    """Forward over bands disjoint from the ones o, lse already hold a
    softmax over; merges into o, lse (the softmax over both sets)."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_fwd_merge(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)), "spa_attn_fwd_merge")
    return o, lse


def spa_attn_bwd_workspace_bytes(B: int, H: int, N: int) -> int:
    return int(_lib.spa_attn_bwd_workspace_bytes(B, H, N))


def spa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, scale: float, lo=None, hi=None,
                 stream=None):
    """Gradients of sum(o * dout): writes dq, dk, dv.  workspace: CUDA tensor of
    at least spa_attn_bwd_workspace_bytes(B, H, N) bytes."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    _need_workspace(workspace, B, H, N)
    s = _stream_ptr(stream)
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv, workspace)]
    if lo is None:
        _check(_lib.spa_attn_bwd(*ptrs, B, H, N, d, scale, s), "spa_attn_bwd")
    else:
        _check(_lib.spa_attn_bwd_ex(*ptrs, B, H, N, d, scale, _i32(lo), _i32(hi), s),
               "spa_attn_bwd_ex")
    return dq, dk, dv


def spa_attn_bwd_fused_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.spa_attn_bwd_fused_workspace_bytes(B, H, N, d))


def spa_attn_bwd_fused(q, k, v, o, dout, lse, dq, dk, dv, workspace, scale: float, lo=None, hi=None,
                       stream=None, steps: int = 7):
    """The backward in one pass over the key tiles (spa_attn_bwd_fused in
    spa.h): same gradients as spa_attn_bwd, dq summed in fp32 by reductions
    (not bit-reproducible from call to call).  workspace: CUDA tensor of at
    least spa_attn_bwd_fused_workspace_bytes(B, H, N, d) bytes."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    if not workspace.is_cuda or not workspace.is_contiguous() or \
            workspace.numel() * workspace.element_size() < spa_attn_bwd_fused_workspace_bytes(B, H, N, d):
        raise ValueError("workspace: contiguous CUDA tensor of spa_attn_bwd_fused_workspace_bytes(B, H, N, d) bytes")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv, workspace)]
    if steps == 7:
        _check(_lib.spa_attn_bwd_fused(*ptrs, B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)),
               "spa_attn_bwd_fused")
    else:  # one or two of its launches (spa_attn_bwd_fused_steps)
        _check(_lib.spa_attn_bwd_fused_steps(*ptrs, B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream), steps),
               "spa_attn_bwd_fused_steps")
    return dq, dk, dv


def attention_backward_fused(q, k, v, o, dout, lse, scale=None, lo=None, hi=None):
    """Allocate dq / dk / dv / workspace and run spa_attn_bwd_fused."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(spa_attn_bwd_fused_workspace_bytes(B, H, N, d) // 4, dtype=torch.float32, device=q.device)
    return spa_attn_bwd_fused(q, k, v, o, dout, lse, dq, dk, dv, ws, scale, lo, hi)


def spa_attn_bwd_stored_workspace_bytes(B: int, H: int, N: int, d: int, lo=None, hi=None) -> int:
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    return int(_lib.spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo_a, hi_a))


def spa_attn_bwd_stored(q, k, v, o, dout, lse, dq, dk, dv, workspace, scale: float, lo=None, hi=None,
                        stream=None, steps: int = 7):
    """The backward that stores dS (spa_attn_bwd_stored in spa.h): same
    gradients as spa_attn_bwd, bit-reproducible; the dK/dV pass writes every
    tile pair's dS^T to the workspace and the dQ pass contracts it with k.
    workspace: CUDA tensor of at least
    spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo, hi) bytes."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    need = spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo, hi)
    if need == 0 or not workspace.is_cuda or not workspace.is_contiguous() or \
            workspace.numel() * workspace.element_size() < need:
        raise ValueError("workspace: contiguous CUDA tensor of spa_attn_bwd_stored_workspace_bytes(B, H, N, d, "
                         "lo, hi) bytes")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv, workspace)]
    if steps == 7:
        _check(_lib.spa_attn_bwd_stored(*ptrs, B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)),
               "spa_attn_bwd_stored")
    else:  # one or two of its launches (spa_attn_bwd_stored_steps)
        _check(_lib.spa_attn_bwd_stored_steps(*ptrs, B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream), steps),
               "spa_attn_bwd_stored_steps")
    return dq, dk, dv


def attention_backward_stored(q, k, v, o, dout, lse, scale=None, lo=None, hi=None):
    """Allocate dq / dk / dv / workspace and run spa_attn_bwd_stored."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo, hi), dtype=torch.uint8, device=q.device)
    return spa_attn_bwd_stored(q, k, v, o, dout, lse, dq, dk, dv, ws, scale, lo, hi)


SPA_NOALLOC_MAX_ROWS = 1 << 20


def spa_attn_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, scale: float, stream=None):
    """Backward without a workspace argument and without any allocation, for
    callers that cannot call cudaMalloc (see spa_attn_bwd_noalloc in spa.h):
    the row sums D go to a library-owned device array of
    SPA_NOALLOC_MAX_ROWS floats, shared by every call -- calls that overlap on
    the GPU race on it.  B * H * N must not exceed SPA_NOALLOC_MAX_ROWS."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv)]
    _check(_lib.spa_attn_bwd_noalloc(*ptrs, B, H, N, d, scale, _stream_ptr(stream)),
           "spa_attn_bwd_noalloc")
    return dq, dk, dv


def _need_workspace(workspace, B, H, N):
    if not workspace.is_cuda or not workspace.is_contiguous() or \
            workspace.numel() * workspace.element_size() < spa_attn_bwd_workspace_bytes(B, H, N):
        raise ValueError("workspace: contiguous CUDA tensor of spa_attn_bwd_workspace_bytes(B, H, N) bytes")


def _need_step(B, H, N, d, tensors, lse=None, workspace=None):
    """The checks spa_attn_bwd makes, for the step entry points: every tensor
    [B, H, N, d] bf16, contiguous, on the GPU; lse [B, H, N] fp32; the
    workspace large enough for D."""
    for t, n in tensors:
        _need(t, (B, H, N, d), torch.bfloat16, n)
    if lse is not None:
        _need(lse, (B, H, N), torch.float32, "lse")
    if workspace is not None:
        _need_workspace(workspace, B, H, N)


def spa_attn_bwd_preprocess(o, dout, workspace, stream=None):
    B, H, N, d = _dims(o)
    _need_step(B, H, N, d, ((o, "o"), (dout, "dout")), workspace=workspace)
    _check(_lib.spa_attn_bwd_preprocess(o.data_ptr(), dout.data_ptr(), workspace.data_ptr(), B, H, N, d,
                                        _stream_ptr(stream)), "spa_attn_bwd_preprocess")


def spa_attn_bwd_dkdv(q, k, v, dout, lse, workspace, dk, dv, scale: float, lo=None, hi=None,
                      stream=None):
    B, H, N, d = _dims(q)
    _need_step(B, H, N, d, ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dk, "dk"), (dv, "dv")), lse,
               workspace)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_bwd_dkdv(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                  lse.data_ptr(), workspace.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)),
           "spa_attn_bwd_dkdv")


def spa_attn_bwd_dq(q, k, v, dout, lse, workspace, dq, scale: float, lo=None, hi=None, stream=None):
    B, H, N, d = _dims(q)
    _need_step(B, H, N, d, ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dq, "dq")), lse, workspace)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_bwd_dq(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                lse.data_ptr(), workspace.data_ptr(), dq.data_ptr(), B, H, N, d, scale,
                                lo_a, hi_a, _stream_ptr(stream)), "spa_attn_bwd_dq")


def spa_attn_bwd_dkdv_add(q, k, v, dout, lse, workspace, dk, dv, scale: float, lo=None, hi=None,
                          stream=None):
    """The dk/dv pass adding to dk, dv instead of overwriting them."""
    B, H, N, d = _dims(q)
    _need_step(B, H, N, d, ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dk, "dk"), (dv, "dv")), lse,
               workspace)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_bwd_dkdv_add(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                      lse.data_ptr(), workspace.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                      B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)),
           "spa_attn_bwd_dkdv_add")


def spa_attn_bwd_dq_add(q, k, v, dout, lse, workspace, dq, scale: float, lo=None, hi=None, stream=None):
    """The dq pass adding to dq instead of overwriting it."""
    B, H, N, d = _dims(q)
    _need_step(B, H, N, d, ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dq, "dq")), lse, workspace)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_bwd_dq_add(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                    lse.data_ptr(), workspace.data_ptr(), dq.data_ptr(), B, H, N, d, scale,
                                    lo_a, hi_a, _stream_ptr(stream)), "spa_attn_bwd_dq_add")


def spa_attn_bwd_dq_delta(q, k, v, o, dout, lse, workspace, dq, scale: float, lo=None, hi=None,
                          stream=None):
    B, H, N, d = _dims(q)
    _need_step(B, H, N, d, ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq")), lse,
               workspace)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_bwd_dq_delta(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      dout.data_ptr(), lse.data_ptr(), workspace.data_ptr(), dq.data_ptr(),
                                      B, H, N, d, scale, lo_a, hi_a, _stream_ptr(stream)),
           "spa_attn_bwd_dq_delta")


def spa_tile_schedule(N: int, H: int, Bq: int, Bk: int, lo=None, hi=None):
    """Host evaluation of the kernels' tile schedule.  Returns a dict of numpy
    arrays: kt_begin/kt_end [H, nqt], tile_class [H, nqt, nkt], qt_begin/qt_end
    [H, nkt]."""
    import numpy as np
    nqt, nkt = -(-N // Bq), -(-N // Bk)
    kb = np.zeros(H * nqt, np.int32)
    ke = np.zeros(H * nqt, np.int32)
    cls = np.zeros(H * nqt * nkt, np.uint8)
    qb = np.zeros(H * nkt, np.int32)
    qe = np.zeros(H * nkt, np.int32)
    p32 = lambda a: a.ctypes.data_as(_i32p)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_tile_schedule(N, H, lo_a, hi_a, Bq, Bk, p32(kb), p32(ke), cls.ctypes.data_as(_u8p),
                                  p32(qb), p32(qe)), "spa_tile_schedule")
    return {"kt_begin": kb.reshape(H, nqt), "kt_end": ke.reshape(H, nqt),
            "tile_class": cls.reshape(H, nqt, nkt), "qt_begin": qb.reshape(H, nkt),
            "qt_end": qe.reshape(H, nkt)}


def spa_tile_classes_device(N: int, H: int, Bq: int, Bk: int, out: torch.Tensor, lo=None, hi=None,
                            stream=None):
    nqt, nkt = -(-N // Bq), -(-N // Bk)
    _need(out, (H, nqt, nkt), torch.uint8, "out")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_tile_classes_device(N, H, lo_a, hi_a, Bq, Bk, out.data_ptr(), _stream_ptr(stream)),
           "spa_tile_classes_device")
    return out


def spa_debug_wait_timeout(limit_ns: int, stream=None):
    """Make one device wait run out of time (see spa.h); check with spa_device_status()."""
    _check(_lib.spa_debug_wait_timeout(limit_ns, _stream_ptr(stream)), "spa_debug_wait_timeout")


def spa_device_status(stream=None) -> int:
    return int(_lib.spa_device_status(_stream_ptr(stream)))


# ------------------------------------------------------------------ conveniences
def attention_forward(q, k, v, scale=None, lo=None, hi=None):
    """Allocate o / lse and run spa_attn_fwd."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    return spa_attn_fwd(q, k, v, o, lse, scale, lo, hi)


def spa_attn_decode_workspace_bytes(B: int, H: int, N: int, d: int, lo=None, hi=None) -> int:
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    return int(_lib.spa_attn_decode_workspace_bytes(B, H, N, d, lo_a, hi_a))


def spa_attn_decode(q, k, v, pos, o, lse, workspace, scale: float, lo=None, hi=None, stream=None):
    """One new token per sequence: q [B, H, d] at positions pos (int32 [B]) of
    the caches k, v [B, H, N, d]; writes o [B, H, d] and lse [B, H]."""
    B, H, N, d = _dims(k)
    _need(k, (B, H, N, d), torch.bfloat16, "k")
    _need(v, (B, H, N, d), torch.bfloat16, "v")
    _need(q, (B, H, d), torch.bfloat16, "q")
    _need(o, (B, H, d), torch.bfloat16, "o")
    _need(lse, (B, H), torch.float32, "lse")
    _need(pos, (B,), torch.int32, "pos")
    if not workspace.is_cuda or not workspace.is_contiguous() or \
            workspace.numel() * workspace.element_size() < spa_attn_decode_workspace_bytes(B, H, N, d, lo, hi):
        raise ValueError("workspace: contiguous CUDA tensor of spa_attn_decode_workspace_bytes(...) bytes")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), pos.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), workspace.data_ptr(), B, H, N, d, scale, lo_a, hi_a,
                                _stream_ptr(stream)), "spa_attn_decode")
    return o, lse


def attention_decode(q, k_cache, v_cache, pos, scale=None, lo=None, hi=None):
    """Allocate o / lse / workspace and run spa_attn_decode."""
    B, H, N, d = _dims(k_cache)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty((B, H, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    nbytes = spa_attn_decode_workspace_bytes(B, H, N, d, lo, hi)
    ws = torch.empty(max(nbytes // 4, 1), dtype=torch.float32, device=q.device)
    return spa_attn_decode(q, k_cache, v_cache, pos, o, lse, ws, scale, lo, hi)


def attention_backward(q, k, v, o, dout, lse, scale=None, lo=None, hi=None):
    """Allocate dq / dk / dv / workspace and run spa_attn_bwd."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device=q.device)
    return spa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, ws, scale, lo, hi)


class SPAttentionFunction(torch.autograd.Function):
    """Band-sparse attention as an autograd function (bf16 [B, H, N, d])."""

    @staticmethod
    def forward(ctx, q, k, v, scale, lo, hi, backward="two-pass"):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = attention_forward(q, k, v, scale, lo, hi)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale, ctx.lo, ctx.hi, ctx.backward = scale, lo, hi, backward
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse = ctx.saved_tensors
        bwd = BACKWARDS[ctx.backward]
        dq, dk, dv = bwd(q, k, v, o, dout.contiguous(), lse, ctx.scale, ctx.lo, ctx.hi)
        return dq, dk, dv, None, None, None, None


BACKWARDS = {"two-pass": attention_backward, "fused": attention_backward_fused,
             "stored": attention_backward_stored}


def spattention(q, k, v, scale=None, lo=None, hi=None, backward: str = "two-pass"):
    """SPAttention: head h of H attends to causal distances in its Balanced
    Distance Partitioning band (or the explicit bands lo/hi).  backward:
    "two-pass" (spa_attn_bwd, deterministic), "fused" (spa_attn_bwd_fused,
    dq summed by fp32 reductions) or "stored" (spa_attn_bwd_stored,
    deterministic, dS kept in a workspace of about 2 bytes per causal pair)."""
    if backward not in BACKWARDS:
        raise ValueError("backward is 'two-pass', 'fused' or 'stored'")
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    return SPAttentionFunction.apply(q, k, v, scale, lo, hi, backward)


# ------------------------------------------------------------- band + shared window
def spa_attn_union_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.spa_attn_union_workspace_bytes(B, H, N, d))


def spa_union_parts(N: int, H: int, window: int, lo=None, hi=None):
    """The two disjoint distance intervals per head that the union calls run:
    returns (a1, b1, a2, b2), lists of H ints."""
    out = [(ctypes.c_int32 * H)() for _ in range(4)]
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_union_parts(N, H, int(window), lo_a, hi_a, *out), "spa_union_parts")
    return tuple(list(a) for a in out)


def _union_ws(workspace, B, H, N, d):
    need = spa_attn_union_workspace_bytes(B, H, N, d)
    if not workspace.is_cuda or workspace.numel() * workspace.element_size() < need:
        raise ValueError("workspace: CUDA tensor of spa_attn_union_workspace_bytes(B, H, N, d) bytes")


def spa_attn_fwd_union(q, k, v, o, lse, scale: float, window: int, lo=None, hi=None, stream=None):
    """Each head attends to its band and to the distances [0, window) that every
    head shares; writes o [B,H,N,d] bf16 and lse [B,H,N] fp32."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    _check(_lib.spa_attn_fwd_union(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   B, H, N, d, scale, int(window), lo_a, hi_a, _stream_ptr(stream)),
           "spa_attn_fwd_union")
    return o, lse


def spa_attn_bwd_union(q, k, v, o, dout, lse, dq, dk, dv, workspace, scale: float, window: int, lo=None,
                       hi=None, stream=None):
    """Gradients of sum(o * dout) for spa_attn_fwd_union (o, lse from it)."""
    B, H, N, d = _dims(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _need(lse, (B, H, N), torch.float32, "lse")
    _union_ws(workspace, B, H, N, d)
    lo_a = None if lo is None else _i32(lo)
    hi_a = None if hi is None else _i32(hi)
    ptrs = [t.data_ptr() for t in (q, k, v, o, dout, lse, dq, dk, dv, workspace)]
    _check(_lib.spa_attn_bwd_union(*ptrs, B, H, N, d, scale, int(window), lo_a, hi_a, _stream_ptr(stream)),
           "spa_attn_bwd_union")
    return dq, dk, dv


def _union_workspace(q):
    B, H, N, d = _dims(q)
    nbytes = spa_attn_union_workspace_bytes(B, H, N, d)
    return torch.empty(max(nbytes // 4, 1), dtype=torch.float32, device=q.device)


def attention_forward_union(q, k, v, window: int, scale=None, lo=None, hi=None):
    """Allocate o / lse and run spa_attn_fwd_union."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    return spa_attn_fwd_union(q, k, v, o, lse, scale, window, lo, hi)


def attention_backward_union(q, k, v, o, dout, lse, window: int, scale=None, lo=None, hi=None):
    """Allocate dq / dk / dv / workspace and run spa_attn_bwd_union."""
    B, H, N, d = _dims(q)
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    return spa_attn_bwd_union(q, k, v, o, dout, lse, dq, dk, dv, _union_workspace(q), scale, window, lo, hi)


class SPAttentionUnionFunction(torch.autograd.Function):
    """Band plus a local window shared by every head, as an autograd function."""

    @staticmethod
    def forward(ctx, q, k, v, window, scale, lo, hi):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = attention_forward_union(q, k, v, window, scale, lo, hi)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.window, ctx.scale, ctx.lo, ctx.hi = window, scale, lo, hi
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attention_backward_union(q, k, v, o, dout.contiguous(), lse, ctx.window, ctx.scale, ctx.lo,
                                              ctx.hi)
        return dq, dk, dv, None, None, None, None


def spattention_union(q, k, v, window: int, scale=None, lo=None, hi=None):
    """Each head attends to its band and to the distances [0, window) that
    every head shares (spa_attn_fwd_union / spa_attn_bwd_union); differentiable."""
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    return SPAttentionUnionFunction.apply(q, k, v, int(window), scale, lo, hi)


def spa_attn_union_merge(o, lse, o2, lse2, stream=None):
    """(o, lse) <- softmax over the union of two disjoint parts' (o, lse), (o2, lse2)."""
    B, H, N, d = _dims(o)
    for t, n in ((o, "o"), (o2, "o2")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    for t, n in ((lse, "lse"), (lse2, "lse2")):
        _need(t, (B, H, N), torch.float32, n)
    _check(_lib.spa_attn_union_merge(o.data_ptr(), lse.data_ptr(), o2.data_ptr(), lse2.data_ptr(), B, H, N, d,
                                     _stream_ptr(stream)), "spa_attn_union_merge")
    return o, lse


def spa_attn_union_add_grads(dq, dk, dv, dq2, dk2, dv2, stream=None):
    """dq += dq2, dk += dk2, dv += dv2 (bf16)."""
    B, H, N, d = _dims(dq)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dq2, "dq2"), (dk2, "dk2"), (dv2, "dv2")):
        _need(t, (B, H, N, d), torch.bfloat16, n)
    _check(_lib.spa_attn_union_add_grads(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dq2.data_ptr(),
                                         dk2.data_ptr(), dv2.data_ptr(), B, H, N, d, _stream_ptr(stream)),
           "spa_attn_union_add_grads")
    return dq, dk, dv
