"""Head sharding with the CUDA op inside: a one-rank NCCL group on cuda:0
(the only multi-GPU form this suite can run) must give exactly the unsharded
spattention output and gradients, since one rank holds every head in order
and the all-to-alls are copies."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

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
    finally:
        dist.destroy_process_group()
