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
    # B4 H32 N8192 d128 by hand: lo_h = 256 h, so the active rows (query rows
    # with a non-empty band, = key rows some query reaches) are
    # 4 * sum_h (8192 - 256 h) = 4 * (32 * 8192 - 256 * 496) = 540672.
    w = synth.WORKLOADS["b4_h32_n8192_d128"]
    bands = ([256 * h for h in range(32)], [256 * (h + 1) for h in range(32)])
    act = bench.active_rows(w, bands)
    assert act == 540672
    pairs = 4 * 8192 * 8193 // 2
    T_act, T_all = 540672 * 128 * 2, 4 * 32 * 8192 * 128 * 2  # bf16 tensors: active rows / every row
    R_act, R_all = 540672 * 4, 4 * 32 * 8192 * 4              # fp32 row vectors
    work = bench.kernel_work(w, pairs, act)
    assert work["spa_fwd_kernel"] == (4 * 128 * pairs, 4 * 128 * pairs, 3 * T_act + T_all + R_all)
    assert work["spa_bwd_dq_kernel"] == (2 * 128 * pairs, 6 * 128 * pairs, 5 * T_act + 2 * R_act + T_all)
    assert work["spa_bwd_dkdv_kernel"] == (8 * 128 * pairs, 8 * 128 * pairs, 4 * T_act + 2 * R_act + 2 * T_all)
    flops, nbytes = bench.step_work(w, pairs, act)
    assert flops == 14 * 128 * pairs
    # the measurement section's figures for this workload: 0.69 GB forward,
    # 1.50 GB backward
    assert round((3 * T_act + T_all + R_all) / 1e9, 2) == 0.69
    assert round((5 * T_act + 2 * R_act + 3 * T_all) / 1e9, 2) == 1.50
    assert nbytes == 8 * T_act + 4 * T_all + R_all + 2 * R_act
    # useful FLOPs over the three kernels of the two-pass step: 4 + 2 + 8 = 14 d
    # per pair; executed 18 d.  The one-pass step executes 14 d.
    two = [work[k] for k in bench.KERNELS_TWO_PASS]
    one = [work[k] for k in bench.KERNELS_FUSED]
    assert sum(u for u, _, _ in two) == sum(u for u, _, _ in one) == 14 * 128 * pairs
    assert sum(e for _, e, _ in two) == 18 * 128 * pairs
    assert sum(e for _, e, _ in one) == 14 * 128 * pairs
    F_act = 540672 * 128 * 4  # the fp32 dq sums over the active rows
    assert work["spa_bwd_fused_kernel"][2] == 4 * T_act + 2 * R_act + 2 * T_all + 2 * F_act
    assert work["spa_bwd_dq_convert_kernel"][2] == F_act + T_act
    # at width 256 every kernel moves more bytes than its useful FLOPs need time
    assert all(bench.roofline_bound(u, b, peaks) == "hbm" for u, _, b in work.values())
    # width-1024 bands (B1 H32 N32768): the forward and dK/dV are tensor-bound,
    # the dQ pass's 2 d useful FLOPs per pair are not
    w = synth.WORKLOADS["b1_h32_n32768_d128"]
    bands = ([1024 * h for h in range(32)], [1024 * (h + 1) for h in range(32)])
    pairs = 32768 * 32769 // 2
    work = bench.kernel_work(w, pairs, bench.active_rows(w, bands))
    assert bench.roofline_bound(work["spa_fwd_kernel"][0], work["spa_fwd_kernel"][2], peaks) == "tensor"
    assert bench.roofline_bound(work["spa_bwd_dkdv_kernel"][0], work["spa_bwd_dkdv_kernel"][2], peaks) == "tensor"
    assert bench.roofline_bound(work["spa_bwd_dq_kernel"][0], work["spa_bwd_dq_kernel"][2], peaks) == "hbm"
    assert bench.roofline_bound(1000.0, 4.0, peaks) == "tensor"
    assert bench.roofline_bound(1000.0, 4.1, peaks) == "hbm"


def test_kernel_report_uses_the_bound_s_algorithmic_work():
    import bench
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    r = bench.kernel_report(1.6e12, 3.2e12, 1e6, 2.0, 0.5, peaks)  # 1.6 TFLOP in 2 ms: tensor-bound
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(800.0) and r["frac"] == pytest.approx(0.5)
    assert r["executed_tflops"] == pytest.approx(1600.0)
    r = bench.kernel_report(1e9, 1e9, 6.4e9, 2.0, 0.5, peaks)  # 6.4 GB in 2 ms: HBM-bound
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3200.0) and r["frac"] == pytest.approx(0.5)


def test_stored_backward_work_counts_every_tile_pair_once():
    # the stored-dS backward writes and reads one bf16 128 x 128 dS^T tile
    # per tile pair the dK/dV pass walks: the pairs holding a permitted
    # element, counted here by the oracle's brute-force tile classes
    import numpy as np

    import bench
    import oracle
    from head_partitioned_distance_b200 import spa, synth
    w = synth.WORKLOADS["b8_h16_n4096_d128"]
    bands = spa.spa_band_bounds(w.N, w.H)
    lo, hi = oracle.bands(w.N, w.H)
    tiles = w.B * int(np.count_nonzero(oracle.tile_classes(w.N, lo, hi, 128, 128)))
    assert bench.stored_tiles(spa, w, bands) == tiles
    pairs = w.B * bench.workload_pairs(w.N, bands)
    act = bench.active_rows(w, bands)
    d = w.d
    T_act, T_all = act * d * 2, w.B * w.H * w.N * d * 2
    work = bench.kernel_work(w, pairs, act, tiles)
    assert work["spa_bwd_dkdv_kernel_ds"][:2] == work["spa_bwd_dkdv_kernel"][:2]
    assert work["spa_bwd_dkdv_kernel_ds"][2] == work["spa_bwd_dkdv_kernel"][2] + tiles * 32768
    assert work["spa_bwd_dq_stored_kernel"] == (2 * d * pairs, 2 * d * tiles * 16384, tiles * 32768 + T_act + T_all)
    assert work["spa_bwd_delta_band_kernel"] == (0, 0, 2 * T_act + act * 4)
    # the three backwards' useful FLOPs agree: 10 d per pair
    useful = lambda ks: sum(work[k][0] for k in ks if k != "spa_fwd_kernel")
    assert useful(bench.KERNELS_STORED) == useful(bench.KERNELS_TWO_PASS) == useful(bench.KERNELS_FUSED) \
        == 10 * d * pairs
