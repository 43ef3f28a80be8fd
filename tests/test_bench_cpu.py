"""bench.py on CPU: the reference arm (the fp64 oracle, the only arm that runs
without a GPU) prints one JSON line with the keys the benchmark contract
names; the CUDA arm refuses to run without a device instead of falling back;
fewer than three warm-up steps are rejected; the DRAM traffic of a kernel is
read from an ncu summary only when the summary names the current sources."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, timeout=300):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    r = _bench("--impl", "reference", "--workload", "b1_h4_n256_d64", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["config"]["workload"] == "b1_h4_n256_d64"
    # the same config keys the CUDA arm prints, so the two lines compare
    import bench
    from head_partitioned_distance_b200 import synth
    w = synth.WORKLOADS["b1_h4_n256_d64"]
    assert line["config"] == bench.spa_config(w, 256 * 257 // 2, 1, False)
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a CUDA device")
@pytest.mark.parametrize("extra", [[], ["--decode"], ["--union", "256"]])
def test_cuda_arm_refuses_to_run_without_a_device(extra):
    r = _bench("--steps", "1", "--warmup", "3", *extra)
    assert r.returncode != 0
    assert "needs a CUDA device" in (r.stdout + r.stderr)


def test_fewer_than_three_warmup_steps_are_rejected():
    r = _bench("--impl", "reference", "--workload", "b1_h4_n256_d64", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr


def test_traffic_is_read_only_from_a_summary_of_the_current_sources(tmp_path, monkeypatch):
    import bench
    csrc = tmp_path / "head_partitioned_distance_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("int k_v1;  // kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_src_sha()
    (tmp_path / "profiles" / "k_w.md").write_text(
        "# summary\n\ntraffic: kernel=spa_k workload=w1 src_sha=%s dram_bytes_per_launch=12345\n" % sha)
    assert bench.ncu_traffic("spa_k", "w1") == 12345.0
    assert bench.ncu_traffic("spa_k", "w2") is None          # another workload
    assert bench.ncu_traffic("spa_other", "w1") is None      # another kernel
    # a comment or layout edit is not a change of the kernel
    (csrc / "k.cuh").write_text("/* the kernel */\n\n   int k_v1;   // first version, reworded\n")
    assert bench.kernel_src_sha() == sha
    assert bench.ncu_traffic("spa_k", "w1") == 12345.0
    (csrc / "k.cuh").write_text("int k_v2;  // kernel v2\n")   # the kernel changed since the capture
    assert bench.kernel_src_sha() != sha
    assert bench.ncu_traffic("spa_k", "w1") is None


def test_gpus_n_starts_n_ranks():
    # --gpus 2 without a torchrun world starts two ranks itself; the dry run
    # takes the launch and reporting path with no GPU work (gloo group,
    # barrier, max over ranks), and rank 0 alone prints the line.
    r = _bench("--gpus", "2", "--dry-run", "--steps", "3", "--warmup", "3", timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(x) for x in r.stdout.strip().splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["dry_run"] is True


def test_gpus_must_match_the_world_it_runs_in():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "world of 1 ranks" in r.stderr


def test_ncu_summaries_from_csv(tmp_path):
    # the summaries under profiles/ are written by these two functions from
    # ncu's CSV output; check them on a tiny hand-made CSV of each kind
    import bench
    raw = tmp_path / "raw.csv"
    hdr = ["ID", "Kernel Name", "gpu__time_duration.sum", "dram__bytes_read.sum", "dram__bytes_write.sum",
           "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
           "smsp__average_warps_issue_stalled_wait_per_issue_active.ratio",
           "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio"]
    units = ["", "", "us", "Mbyte", "Gbyte", "%", "inst", "inst"]
    vals = ["0", "void spa_k<128>(CUtensorMap_st)", "12.5", "500", "0.25", "51.5", "1.5", "2.5"]
    raw.write_text("\n".join(",".join(f'"{x}"' for x in r) for r in (hdr, units, vals)) + "\n")
    md = bench.ncu_summary(str(raw), "spa_k", "w1", "ncu ...", "abc123")
    assert "traffic: kernel=spa_k workload=w1 src_sha=abc123 dram_bytes_per_launch=750000000" in md
    assert "51.5 %" in md and "long_scoreboard 2.50, wait 1.50" in md
    ll = tmp_path / "ll.csv"
    rows = [["ID", "Kernel Name", "Metric Name", "Metric Value"]]
    for i, (k, ns) in enumerate([("a", 300), ("b", 100), ("a", 300), ("b", 300)]):
        rows.append([str(i), f"void spa_{k}_kernel<128>(x)", "gpu__time_duration.sum", str(ns)])
    ll.write_text("==PROF== noise\n" + "\n".join(",".join(f'"{x}"' for x in r) for r in rows) + "\n")
    md = bench.ncu_launch_list(str(ll), "w1", "ncu ...")
    assert "| spa_a_kernel<128> | 2 | 0.6 | 60.0 % |" in md
    assert "| spa_b_kernel<128> | 2 | 0.4 | 40.0 % |" in md
    # the dK/dV pass that stores dS has its own key in the bench line
    assert bench.bench_kernel_key("spa_bwd_dkdv_kernel<128, 0, 1>") == "spa_bwd_dkdv_kernel_ds"
    assert bench.bench_kernel_key("spa_bwd_dkdv_kernel<128, 0, 0>") == "spa_bwd_dkdv_kernel"
    assert bench.bench_kernel_key("spa_fwd_kernel<128, 0, 1>") == "spa_fwd_kernel"


def test_backward_modes_are_consistent():
    # every backward the bench can time has a kernel list, a description and
    # a work entry for each kernel it launches (the line's per-kernel roofline)
    import bench
    from head_partitioned_distance_b200 import synth
    modes = {"two-pass", "stored", "fused"}
    assert set(bench.KERNELS_OF) == set(bench.BACKWARD_DESCRIPTION) == modes
    w = synth.WORKLOADS["b1_h8_n1001_d64"]
    work = bench.kernel_work(w, 1000, 500, 10)
    for mode, kernels in bench.KERNELS_OF.items():
        assert kernels[0] == "spa_fwd_kernel", mode
        for k in kernels:
            assert k in work, (mode, k)
