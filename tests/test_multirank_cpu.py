"""The benchmark's multi-rank host logic on CPU: two gloo ranks take the max
of their timings and aggregate whole-job throughput the way bench.py does
under torchrun (each rank an independent batch, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, local, w = bench.dist_setup()
    assert (r, local, w) == (rank, rank, world)
    d = bench.dist_init("gloo", local)
    try:
        elapsed = [120.0, 150.0][rank]          # this rank's device time for K steps (ms)
        mx = bench.reduce_max(elapsed, torch.device("cpu"))
        value = bench.aggregate(1e12, 10, world, mx)
        d.barrier()
        q.put((rank, mx, value))
    finally:
        d.destroy_process_group()


def test_two_gloo_ranks_max_time_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, value in got:
        assert mx == 150.0
        # 2 ranks x 1e12 flops x 10 steps over the slowest rank's 150 ms
        assert value == pytest.approx(2 * 1e12 * 10 / 0.150 / 1e12)


def test_band_pair_counting_matches_oracle():
    import bench
    import oracle
    for N, H in [(256, 4), (1001, 8), (777, 5)]:
        lo, hi = oracle.bands(N, H)
        want = sum(oracle.band_pairs(N, int(a), int(b)) for a, b in zip(lo, hi))
        assert bench.workload_pairs(N, (lo.tolist(), hi.tolist())) == want == N * (N + 1) // 2
    # prefix counts used by the CPU-baseline sample
    assert bench.band_pairs_prefix(10, 0, 4) == sum(min(i + 1, 4) for i in range(10))


def test_kernel_work_and_roofline_bound():
    import bench
    from head_partitioned_distance_b200 import synth
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}  # ridge point 250 FLOP per byte
    w = synth.WORKLOADS["b1_h32_n32768_d128"]
    pairs = w.B * w.N * (w.N + 1) // 2  # the bands partition the causal distances
    work = bench.kernel_work(w, pairs)
    T, R = w.B * w.H * w.N * w.d * 2, w.B * w.H * w.N * 4
    # S and dP run in both backward passes: 18 d per pair executed, 14 d useful
    assert sum(f for f, _ in work.values()) == 18 * w.d * pairs
    assert sum(b for _, b in work.values()) == 16 * T + 5 * R
    assert bench.step_work(w, pairs) == (14 * w.d * pairs, 12 * T + 2 * R)
    # width-1024 bands: about 4 d W FLOPs against 8 d bytes per row in the forward
    assert all(bench.roofline_bound(f, b, peaks) == "tensor" for f, b in work.values())
    # width-256 bands at d = 128 move more bytes than the tensor cores need time for
    w = synth.WORKLOADS["b8_h16_n4096_d128"]
    work = bench.kernel_work(w, w.B * w.N * (w.N + 1) // 2)
    assert bench.roofline_bound(*work["spa_fwd_kernel"], peaks) == "hbm"
    assert bench.roofline_bound(1000.0, 4.0, peaks) == "tensor"
    assert bench.roofline_bound(1000.0, 4.1, peaks) == "hbm"
