"""Head sharding (head_partitioned_distance_b200/sharding.py) on CPU: the pair
assignment and its balance, and -- with 2 and 4 gloo ranks -- the
sequence <-> head all-to-all and sequence-parallel attention, whose output and
gradients must equal the oracle's on the unsharded tensors.  The attention
inside each rank is the fp64 oracle (spa_fwd / spa_bwd with the rank's heads
and their global bands) wrapped as an autograd function, since the CUDA op
needs a GPU: these tests check the sharding and the exchange against the
oracle's whole-batch result, not the kernel."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from head_partitioned_distance_b200 import sharding


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _OracleAttention(torch.autograd.Function):
    """The oracle's band attention on [B, Hl, N, d] fp64 CPU tensors, head i
    with band [lo[i], hi[i]); the backward is the oracle's gradient of
    sum(o * dout)."""

    @staticmethod
    def forward(ctx, q, k, v, scale, lo, hi):
        ctx.save_for_backward(q, k, v)
        ctx.scale, ctx.lo, ctx.hi = scale, lo, hi
        o, _ = oracle.spa_fwd(q.numpy(), k.numpy(), v.numpy(), scale, lo, hi)
        return torch.from_numpy(o)

    @staticmethod
    def backward(ctx, dout):
        q, k, v = ctx.saved_tensors
        grads = oracle.spa_bwd(q.numpy(), k.numpy(), v.numpy(), dout.contiguous().numpy(), ctx.scale,
                               ctx.lo, ctx.hi)
        return tuple(torch.from_numpy(g) for g in grads) + (None, None, None)


def oracle_attention(q, k, v, scale=None, lo=None, hi=None):
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    return _OracleAttention.apply(q.contiguous(), k.contiguous(), v.contiguous(), scale,
                                  [int(x) for x in lo], [int(x) for x in hi])


# ------------------------------------------------------------------ assignment
@pytest.mark.parametrize("H,world", [(32, 8), (32, 4), (32, 2), (8, 4), (2, 1)])
def test_paired_heads_cover_every_head_once_in_pairs(H, world):
    hs = sharding.paired_heads(H, world)
    assert len(hs) == world
    assert sorted(h for r in hs for h in r) == list(range(H))
    for r in hs:
        assert len(r) == H // world
        assert all((H - 1 - h) in r for h in r)


def test_paired_heads_reject_uneven_splits():
    for H, world in [(30, 4), (7, 1), (32, 3)]:
        with pytest.raises(ValueError):
            sharding.paired_heads(H, world)


def test_pairing_balances_the_work_and_contiguous_blocks_do_not():
    N, H = 32768, 32
    lo, hi = oracle.bands(N, H)
    assert sharding.band_bounds(N, H) == ([int(x) for x in lo], [int(x) for x in hi])
    for h in (0, 5, 31):
        assert sharding.head_pairs(N, int(lo[h]), int(hi[h])) == oracle.band_pairs(N, int(lo[h]), int(hi[h]))
    for world in (2, 4, 8):
        per = sharding.rank_pairs(N, H, world)
        assert max(per) == min(per)  # lo_h + lo_{H-1-h} is the same for every h here
        contiguous = [sum(sharding.head_pairs(N, int(lo[h]), int(hi[h]))
                          for h in range(r * H // world, (r + 1) * H // world)) for r in range(world)]
        assert max(contiguous) / min(contiguous) > 1.5


# ------------------------------------------------------------------ gloo ranks
def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 2, 8, 48, 4
        g = torch.Generator().manual_seed(0)
        full = [torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4)]  # q k v dout
        n = N // world
        chunk = lambda t: t[:, :, rank * n:(rank + 1) * n].contiguous()
        heads = sharding.paired_heads(H, world)
        # exchange: content and round trip
        xh = sharding.seq_to_heads(chunk(full[0]), heads)
        assert torch.equal(xh, full[0][:, heads[rank]])
        assert torch.equal(sharding.heads_to_seq(xh, heads), chunk(full[0]))
        # sequence-parallel attention against the oracle on the whole batch
        ql, kl, vl = (chunk(t).requires_grad_(True) for t in full[:3])
        o = sharding.sequence_parallel_attention(ql, kl, vl, H, scale=0.3, attn_fn=oracle_attention)
        (o * chunk(full[3])).sum().backward()
        qn, kn, vn, dn = (t.numpy() for t in full)
        of, _ = oracle.spa_fwd(qn, kn, vn, 0.3)
        gq, gk, gv = oracle.spa_bwd(qn, kn, vn, dn, 0.3)
        errs = [(o - chunk(torch.from_numpy(of))).abs().max().item()]
        # each token's gradient comes back to the rank that holds the token
        for gl, gf in ((ql.grad, gq), (kl.grad, gk), (vl.grad, gv)):
            errs.append((gl - chunk(torch.from_numpy(gf))).abs().max().item())
        q.put((rank, errs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sequence_parallel_attention_equals_the_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for _ in range(world):
        rank, errs = q.get(timeout=10)
        assert max(errs) < 1e-12, (rank, errs)


def test_exchanges_reject_shapes_that_do_not_split_over_the_group(monkeypatch):
    # checked before any collective, so no process group is needed
    monkeypatch.setattr(sharding, "_group_size", lambda group: 2)
    heads = sharding.paired_heads(4, 2)
    with pytest.raises(ValueError):
        sharding.heads_to_seq(torch.zeros(1, 2, 7, 4), heads)        # 7 tokens over 2 ranks
    with pytest.raises(ValueError):
        sharding.heads_to_seq(torch.zeros(1, 3, 8, 4), heads)        # 3 local heads, 2 listed per rank
    with pytest.raises(ValueError):
        sharding.seq_to_heads(torch.zeros(1, 4, 4, 4), heads[:1])    # one rank's heads for a group of 2
