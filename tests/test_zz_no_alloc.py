"""The backward entry point that allocates nothing (spa_attn_bwd_noalloc).

Some callers cannot call cudaMalloc -- a plugin inside a host framework that
owns all device memory through its own pool, or a caller that must not risk
the device-wide synchronisation an allocation may cause -- so the library
offers a backward that takes no workspace and keeps its scratch (the row sums
D) in a static device array of SPA_NOALLOC_MAX_ROWS floats.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes both alone in a
fresh process and after the rest of the suite (the scratch array keeps the
previous call's contents, which the entry point must not depend on)."""
import ctypes
import math

import pytest
import torch

from head_partitioned_distance_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from head_partitioned_distance_b200 import spa as mod
    return mod


def _noalloc(spa, q, k, v, o, do, lse, dq, dk, dv, scale):
    """Call the C entry point directly through ctypes."""
    B, H, N, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptrs = [t.data_ptr() for t in (q, k, v, o, do, lse, dq, dk, dv)]
    return spa._lib.spa_attn_bwd_noalloc(*ptrs, B, H, N, d, ctypes.c_float(scale), stream)


def _case(spa, B, H, N, d, seed):
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in synth.make_inputs(B, H, N, d, seed=seed))
    scale = 1 / math.sqrt(d)
    o, lse = spa.attention_forward(q, k, v, scale)
    return q, k, v, o, do, lse, scale


@pytest.mark.parametrize("B,H,N,d", [(1, 8, 1001, 64), (2, 4, 777, 128), (1, 32, 32768, 128)])
def test_noalloc_backward_matches_workspace_backward_twice(spa, B, H, N, d):
    # Both entry points run the same two kernels on the same D, so the
    # gradients must be bit-identical.  The first no-allocation call runs on
    # other inputs of the same shape, so the scratch array holds a different D
    # when the second call starts: the second call is right only if it writes
    # every D value it reads.
    first = _case(spa, B, H, N, d, seed=97 + N)
    second = _case(spa, B, H, N, d, seed=31 + N)
    for call, (q, k, v, o, do, lse, scale) in enumerate((first, second)):
        ref = spa.attention_backward(q, k, v, o, do, lse, scale)
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        assert _noalloc(spa, q, k, v, o, do, lse, dq, dk, dv, scale) == spa.SPA_OK
        torch.cuda.synchronize()
        assert spa.spa_device_status() == spa.SPA_OK
        for got, want, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            assert torch.equal(got, want), (call, name)


def test_noalloc_rejects_sizes_beyond_its_scratch(spa):
    assert spa.SPA_NOALLOC_MAX_ROWS == 1 << 20
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check fails first
    B, H, N = 1, 32, (1 << 15) + 1   # B * H * N = SPA_NOALLOC_MAX_ROWS + 32
    st = spa._lib.spa_attn_bwd_noalloc(*([fake] * 9), B, H, N, 128, ctypes.c_float(0.1), None)
    assert st == spa.SPA_ERR_UNSUPPORTED
