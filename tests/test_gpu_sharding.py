"""Head sharding with the CUDA op inside: a one-rank NCCL group on cuda:0
(the only multi-GPU form this suite can run) must give exactly the unsharded
spattention output and gradients, since one rank holds every head in order
and the all-to-alls are copies, and both must match the fp64 oracle within
the parity tolerances."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from head_partitioned_distance_b200 import synth

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_one_rank_sequence_parallel_attention_is_spattention():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from head_partitioned_distance_b200 import sharding, spa
    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        B, H, N, d = 1, 8, 1024, 64
        q, k, v, do = (t.to("cuda:0") for t in synth.make_inputs(B, H, N, d, seed=3))
        qs, ks, vs = (t.clone().requires_grad_(True) for t in (q, k, v))
        o = sharding.sequence_parallel_attention(qs, ks, vs, H, scale=0.125)
        (o.float() * do.float()).sum().backward()
        qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
        orf = spa.spattention(qr, kr, vr, scale=0.125)
        (orf.float() * do.float()).sum().backward()
        torch.cuda.synchronize()
        assert spa.spa_device_status() == spa.SPA_OK
        assert torch.equal(o, orf)
        for a, b in ((qs.grad, qr.grad), (ks.grad, kr.grad), (vs.grad, vr.grad)):
            assert torch.equal(a, b)
        # the sharded run against the oracle (the gradient of sum(o * do))
        f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
        qf, kf, vf, dof = (f64(t) for t in (q, k, v, do))
        o_ref, _ = oracle.spa_fwd(qf, kf, vf, 0.125)
        assert np.abs(f64(o) - o_ref).max() <= 2e-2
        for g, ref in zip((qs.grad, ks.grad, vs.grad), oracle.spa_bwd(qf, kf, vf, dof, 0.125)):
            assert np.abs(f64(g) - ref).max() / np.abs(ref).max() <= 5e-2
    finally:
        dist.destroy_process_group()
