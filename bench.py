#!/usr/bin/env python
"""Benchmark: SPAttention band-sparse attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl spa|reference]
                    [--decode | --union W]

One step = one pass of the whole hot path over one batch of synthetic input:
spa_attn_fwd (1 kernel) then the backward (by default spa_attn_bwd_stored: the
row sums D, the dK/dV pass, which also stores each tile pair's dS^T, and the dQ
pass from the stored tiles; see --bwd).  Inputs are resident in HBM
when the timed region starts;
each of q, k, v, dout is larger than the 126 MB L2, so no flush is needed
between steps.  The metric is useful TFLOP/s: 14 * d * (permitted pairs) per
step (forward 4 d, backward 10 d per pair -- the two GEMMs of the forward and
the five of the backward, over the band's pairs only, never the tile padding),
over the device time of the K timed steps, max over ranks.

After the headline measurement, a one-GPU run also times every other
workload of the scope table and the same kernels with full bands (dense causal
attention on every head), a few steps each, and adds them to the line as
"per_workload" (ms per step, useful TFLOP/s, % of the bf16 peak, tokens/s,
fraction of the step roofline); --no-sweep skips it.

N > 1 (torchrun, one process per GPU): every rank runs its own independent
batch of the same workload (weak scaling); the only collectives are the
barrier and the max of the timings.  --gpus N without torchrun starts the N
ranks itself.

The step's backward is the one that stores dS (spa_attn_bwd_stored: D, the
dK/dV pass writing each tile pair's dS^T, the dQ pass contracting it with k);
--bwd two-pass times the two-pass backward (spa_attn_bwd: the dQ pass
computing S and dP again) and --bwd fused the one-pass backward
(spa_attn_bwd_fused) instead.

--impl reference times the fp64 CPU oracle (the slow, plain implementation the
tests check against) on a bounded sample of the same workload and prints the
same line with "impl": "reference".

--decode times the decode step instead (one new token per sequence against a
KV cache, HBM roofline); --union W times the band plus a local window [0, W)
shared by every head (spa_attn_fwd_union + spa_attn_bwd_union), useful FLOPs
over the union's pairs.
"""
from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from head_partitioned_distance_b200 import synth  # noqa: E402

METRIC = "band-sparse attn fwd+bwd useful TFLOP/s and % of B200 bf16 tensor peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "b1_h32_n32768_d128"
L2_BYTES = 126 * 2**20
HOST_LEAD_CYCLES = 400_000  # about 0.2 ms at the B200's clocks
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# one step = the forward, then the backward, in launch order.  Two-pass
# backward: the dQ pass (which also forms the row sums D) and the dK/dV pass.
# One-pass backward: D and the zeroed fp32 dq sums, the pass over key tiles,
# and dq from the sums.
KERNELS_TWO_PASS = ("spa_fwd_kernel", "spa_bwd_dq_kernel", "spa_bwd_dkdv_kernel")
KERNELS_FUSED = ("spa_fwd_kernel", "spa_bwd_fused_prep_kernel", "spa_bwd_fused_kernel", "spa_bwd_dq_convert_kernel")
# Backward that stores dS: D over the reached query tiles, the dK/dV pass that
# also writes each tile pair's dS^T (the DS instantiation of
# spa_bwd_dkdv_kernel, named spa_bwd_dkdv_kernel_ds here), and the dQ pass
# from the stored tiles.
KERNELS_STORED = ("spa_fwd_kernel", "spa_bwd_delta_band_kernel", "spa_bwd_dkdv_kernel_ds", "spa_bwd_dq_stored_kernel")
KERNELS_OF = {"two-pass": KERNELS_TWO_PASS, "fused": KERNELS_FUSED, "stored": KERNELS_STORED}
STORED_TILE_BYTES = 128 * 128 * 2


# --------------------------------------------------------------------- counting
def band_pairs_prefix(P: int, lo: int, hi: int) -> int:
    """Permitted pairs among query rows [0, P) of a head with band [lo, hi):
    distance delta occurs in max(0, P - delta) rows."""
    return sum(max(0, P - dd) for dd in range(lo, hi))


def workload_pairs(N: int, bands) -> int:
    return sum(band_pairs_prefix(N, lo, hi) for lo, hi in zip(*bands))


def union_pairs(N: int, window: int, bands) -> int:
    """Pairs of the band-plus-shared-window sets: distances [0, window) and
    [lo_h, hi_h), each distance counted once."""
    total = 0
    for lo, hi in zip(*bands):
        total += band_pairs_prefix(N, 0, window) + band_pairs_prefix(N, lo, hi)
        a, b = max(0, lo), min(window, hi)
        if b > a:
            total -= band_pairs_prefix(N, a, b)
    return total


def active_rows(w, bands) -> int:
    """act = sum over (b, h) of N - lo_h: the query rows whose band is not
    empty, which equals the number of key rows some query reaches."""
    return w.B * sum(w.N - int(lo) for lo in bands[0])


def kernel_work(w, pairs: int, act: int, tiles: int = 0):
    """Algorithmic work per launch of each kernel, the accounting of the
    scope table's measurement section: (useful FLOPs, executed FLOPs, least
    bytes).  Inputs are counted over the active rows only (head h never reads
    query rows i < lo_h nor key rows j > N - 1 - lo_h); outputs over every
    row (every element is written).  T_act / T_all: one [B, H, N, d] bf16
    tensor over the active / all rows; R_act / R_all: one fp32 row vector
    (lse or D).  The dQ pass executes S, dP and dQ (6 d per pair) but only
    dQ is work the dK/dV pass does not already do, so its useful FLOPs are
    2 d per pair.  `tiles` is the number of 128 x 128 tile pairs the dK/dV
    pass walks (stored_tiles): the stored-dS backward writes and reads one
    bf16 dS^T tile for each, and its dQ pass executes 2 d per element of
    those tiles."""
    d = w.d
    rows = w.B * w.H * w.N
    T_all, T_act, R_all, R_act = rows * d * 2, act * d * 2, rows * 4, act * 4
    F_act = act * d * 4  # one fp32 [B, H, N, d] buffer over the active rows
    return {
        # q k v in over active rows; o, lse out for every row
        "spa_fwd_kernel": (4 * d * pairs, 4 * d * pairs, 3 * T_act + T_all + R_all),
        # one-pass backward: o dO in, D out, fp32 dq sums zeroed over the
        # active rows; dq zeroed on the others
        "spa_bwd_fused_prep_kernel": (0, 0, 2 * T_act + R_act + F_act + (T_all - T_act)),
        # S^T, dP^T, dV, dK, dQ: q k v dO lse D in over active rows, dk dv out
        # for every row, the fp32 dq sums read and written once
        "spa_bwd_fused_kernel": (10 * d * pairs, 10 * d * pairs, 4 * T_act + 2 * R_act + 2 * T_all + 2 * F_act),
        # dq from the sums over the active rows
        "spa_bwd_dq_convert_kernel": (0, 0, F_act + T_act),
        # q k v o dO and lse in over active rows; dq out for every row, D out
        "spa_bwd_dq_kernel": (2 * d * pairs, 6 * d * pairs, 5 * T_act + 2 * R_act + T_all),
        # q k v dO, lse and D in over active rows; dk dv out for every row
        "spa_bwd_dkdv_kernel": (8 * d * pairs, 8 * d * pairs, 4 * T_act + 2 * R_act + 2 * T_all),
        # stored-dS backward: o dO in and D out over the active rows
        "spa_bwd_delta_band_kernel": (0, 0, 2 * T_act + R_act),
        # the dK/dV pass, plus every tile pair's dS^T out
        "spa_bwd_dkdv_kernel_ds": (8 * d * pairs, 8 * d * pairs,
                                   4 * T_act + 2 * R_act + 2 * T_all + tiles * STORED_TILE_BYTES),
        # dS^T tiles and k over active rows in, dq out for every row
        "spa_bwd_dq_stored_kernel": (2 * d * pairs, 2 * d * tiles * 128 * 128,
                                     tiles * STORED_TILE_BYTES + T_act + T_all),
    }


def stored_tiles(spa, w, bands) -> int:
    """Tile pairs (key tile, query tile) the dK/dV pass walks over the whole
    workload: the lengths of its query strips, from the library's schedule."""
    sch = spa.spa_tile_schedule(w.N, w.H, 128, 128, bands[0], bands[1])
    lens = sch["qt_end"] - sch["qt_begin"] + 1
    return w.B * int(lens[lens > 0].sum())


def step_work(w, pairs: int, act: int):
    """(useful FLOPs, least bytes) of one forward + backward step: 14 d per
    pair (the forward's two GEMMs, the backward's five), and the scope
    table's bytes -- forward: q k v over active rows in, o lse out for every
    row; backward: q k v o dO over active rows in, lse and D over active rows,
    dq dk dv out for every row."""
    rows = w.B * w.H * w.N
    d = w.d
    T_all, T_act, R_all, R_act = rows * d * 2, act * d * 2, rows * 4, act * 4
    fwd = 3 * T_act + T_all + R_all
    bwd = 5 * T_act + 2 * R_act + 3 * T_all
    return 14 * d * pairs, fwd + bwd


def roofline_bound(flops: float, nbytes: float, peaks) -> str:
    """"tensor" when the FLOPs at the bf16 peak take longer than the bytes at
    the HBM peak, else "hbm" (the attainable-performance roofline)."""
    return "tensor" if flops / (peaks["bf16_tflops"] * 1e12) >= nbytes / (peaks["hbm_gbs"] * 1e9) else "hbm"


def kernel_report(useful: float, executed: float, nbytes: float, avg_ms: float, share: float, peaks):
    """One kernel against its roofline.  The bound compares the kernel's
    useful FLOPs at the bf16 peak with its least bytes at the HBM peak;
    "achieved" is the algorithmic work of that bound (useful FLOPs or least
    bytes) over the kernel's average launch time.  The executed FLOPs
    (recomputation included) are reported beside it."""
    bound = roofline_bound(useful, nbytes, peaks)
    sec = avg_ms * 1e-3
    if bound == "tensor":
        achieved, peak, unit, units = useful / sec / 1e12, peaks["bf16_tflops"], "TFLOP/s", useful
    else:
        achieved, peak, unit, units = nbytes / sec / 1e9, peaks["hbm_gbs"], "GB/s", nbytes
    return {"bound": bound, "avg_ms": avg_ms, "share": share, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "algorithmic_per_launch": units,
            "useful_flops_per_launch": useful, "executed_flops_per_launch": executed,
            "bytes_per_launch": nbytes,
            "useful_tflops": useful / sec / 1e12, "executed_tflops": executed / sec / 1e12,
            "frac_useful_of_bf16_peak": useful / sec / 1e12 / peaks["bf16_tflops"],
            "frac_executed_of_bf16_peak": executed / sec / 1e12 / peaks["bf16_tflops"],
            "gbs": nbytes / sec / 1e9, "frac_of_hbm_peak": nbytes / sec / 1e9 / peaks["hbm_gbs"]}


def step_roofline_report(step_flops: float, step_bytes: float, step_ms: float, peaks):
    t_flops = step_flops / (peaks["bf16_tflops"] * 1e12) * 1e3
    t_bytes = step_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    return {"bound": "tensor" if t_flops >= t_bytes else "hbm", "flops": step_flops, "bytes": step_bytes,
            "t_flops_ms": t_flops, "t_bytes_ms": t_bytes, "t_measured_ms": step_ms,
            "frac": max(t_flops, t_bytes) / step_ms}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def _code_only(src: str) -> str:
    """Source text with comments and blank lines removed and each line's
    surrounding whitespace stripped: what the compiler sees of it, so that an
    edit of a comment does not count as a change of the kernels."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).strip() for line in src.splitlines())
    return "\n".join(line for line in lines if line)


def kernel_src_sha() -> str:
    """Hash of the kernel sources' code (comments and layout ignored)."""
    csrc = os.path.join(ROOT, "head_partitioned_distance_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary under
    profiles/, when the summary was taken on the current kernel sources."""
    prof = os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    sha = kernel_src_sha()
    for name in sorted(os.listdir(prof)):
        if not name.endswith((".md", ".txt")):
            continue
        fields = {}
        with open(os.path.join(prof, name)) as f:
            for line in f:
                if line.startswith("traffic:"):
                    for kv in line[len("traffic:"):].split():
                        if "=" in kv:
                            a, b = kv.split("=", 1)
                            fields[a] = b
                    if (fields.get("kernel") == kernel and fields.get("workload") == workload
                            and fields.get("src_sha") == sha):
                        return float(fields["dram_bytes_per_launch"])
    return None


# --------------------------------------------------------------------- ncu summaries
_NCU_UNITS = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
_NCU_ROWS = [
    ("gpu__time_duration.sum", "duration (serialised, under ncu)"),
    ("sm__cycles_elapsed.avg.per_second", "SM clock under ncu"),
    ("dram__bytes_read.sum", "DRAM bytes read"),
    ("dram__bytes_write.sum", "DRAM bytes written"),
    ("gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed", "DRAM throughput, % of peak"),
    ("sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active", "tensor pipe active, % of active cycles"),
    ("sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed", "tensor pipe active, % of elapsed cycles"),
    ("smsp__issue_active.avg.pct_of_peak_sustained_active", "issue active, % of peak"),
    ("lts__throughput.avg.pct_of_peak_sustained_elapsed", "L2 throughput, % of peak"),
    ("sm__warps_active.avg.pct_of_peak_sustained_active", "warps active, % of peak"),
    ("launch__registers_per_thread", "registers per thread at launch"),
]


def ncu_summary(csv_path: str, kernel: str, workload: str, command: str, src_sha: str, note: str = "") -> str:
    """Markdown summary of one captured launch from `ncu -i REP --page raw
    --csv` output: the metrics the roofline uses (DRAM bytes, tensor-pipe and
    issue activity, L2 and DRAM throughput), the three largest warp stall
    reasons, and the `traffic:` line that bench.py reads back (DRAM bytes
    read + written by the launch, tagged with the kernel sources' hash)."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    start = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr, units = rows[start], rows[start + 1]
    ki = hdr.index("Kernel Name")
    data = [r for r in rows[start + 2:]
            if len(r) == len(hdr) and bench_kernel_key(r[ki].split("(")[0].replace("void ", "")) == kernel]
    if len(data) != 1:
        raise SystemExit(f"{csv_path}: expected one launch of {kernel}, found {len(data)}")
    rec = dict(zip(hdr, data[0]))
    unit = dict(zip(hdr, units))

    def val(name):
        return float(rec[name].replace(",", ""))

    dram = {}
    for name in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
        dram[name] = val(name) * _NCU_UNITS.get(unit[name], 1.0)
    lines = [f"# ncu --set full -- {rec['Kernel Name'].split('(')[0]}, workload {workload}", "",
             "Command (after the same command exited 0 without ncu; one kernel, one launch):", "",
             f"    {command}", ""]
    if note:
        lines += [note, ""]
    lines += ["| metric | value |", "|---|---|"]
    for name, desc in _NCU_ROWS:
        if name in rec and rec[name] != "":
            lines.append(f"| {desc} (`{name}`) | {rec[name]} {unit[name]} |")
    stalls = sorted(((val(h), h) for h in hdr if h.startswith("smsp__average_warps_issue_stalled_")
                     and h.endswith("_per_issue_active.ratio") and rec.get(h, "") != ""
                     and "selected" not in h), reverse=True)[:3]
    lines.append("| top stalls per issued instruction | " + ", ".join(
        f"{h[len('smsp__average_warps_issue_stalled_'):-len('_per_issue_active.ratio')]} {v:.2f}" for v, h in stalls)
        + " |")
    total = dram["dram__bytes_read.sum"] + dram["dram__bytes_write.sum"]
    lines += ["", f"DRAM bytes per launch (read + written): {total / 1e9:.4f} GB.", "",
              f"traffic: kernel={kernel} workload={workload} src_sha={src_sha} dram_bytes_per_launch={int(total)}"]
    return "\n".join(lines) + "\n"


def bench_kernel_key(ncu_name: str) -> str:
    """The bench line's key of a kernel that ncu names with its template
    arguments: the base name, except the dK/dV pass that stores dS (third
    template argument 1) is spa_bwd_dkdv_kernel_ds."""
    base = ncu_name.split("<")[0].strip()
    args = ncu_name[len(base):].strip("<> ").split(",")
    if base == "spa_bwd_dkdv_kernel" and len(args) == 3 and args[2].strip() in ("1", "true"):
        return "spa_bwd_dkdv_kernel_ds"
    return base


def ncu_launch_list(csv_path: str, workload: str, command: str, bench_json: str = "", note: str = "") -> str:
    """Markdown launch list from `ncu --metrics gpu__time_duration.sum --csv`
    output: per kernel its launches, total time and share under ncu (cold
    cache, serialised), beside the shares of the same kernels in a bench line
    (CUDA events), which are what the ncu shares should agree with."""
    import csv
    rows = [r for r in csv.reader(l for l in open(csv_path) if l.startswith('"'))]
    hdr = rows[0]
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    tot = {}
    for r in rows[1:]:
        if r[mi] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0].replace("void ", "")
        n, t = tot.get(name, (0, 0.0))
        tot[name] = (n + 1, t + float(r[vi].replace(",", "")) * 1e-3)  # ns -> us
    all_us = sum(t for _, t in tot.values())
    bench = {}
    if bench_json:
        line = json.loads(open(bench_json).read().strip().splitlines()[-1])
        bench = line.get("kernels", {})
    lines = [f"# ncu launch list -- bench step, workload {workload}", "",
             "Command (after the same command exited 0 without ncu):", "", f"    {command}", ""]
    if note:
        lines += [note, ""]
    lines += ["| kernel | launches | total us (ncu) | share (ncu) | bench avg ms (events) | share (bench events) |",
              "|---|---|---|---|---|---|"]
    for name, (n, t) in tot.items():
        b = bench.get(bench_kernel_key(name), {})
        bms = f"{b['avg_ms']:.4f}" if b else "-"
        bsh = f"{100 * b['share']:.1f} %" if b else "-"
        lines.append(f"| {name} | {n} | {t:.1f} | {100 * t / all_us:.1f} % | {bms} | {bsh} |")
    lines += ["", f"Kernel sources: src_sha={kernel_src_sha()}."]
    return "\n".join(lines) + "\n"


# --------------------------------------------------------------------- clocks
# NVML clock-event reason bits (nvmlClocksEventReason*)
_NVML_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled every
    `period_s` by a host thread through NVML (reading only) while the timed
    region runs, so that even a region of a few tens of milliseconds holds
    samples.  Falls back to `nvidia-smi -lms 100` when NVML is unavailable."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, torch_device=None, period_s: float = 0.002):
        self.gpu_index = gpu_index
        self.torch_device = torch_device
        self.period_s = period_s
        self.proc = None
        self.thread = None
        self.samples = []  # (perf_counter, sm_mhz, sm_max_mhz, power_w, reason bits)
        self.t0 = self.t1 = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.torch_device is not None:
            props = torch.cuda.get_device_properties(self.torch_device)
            try:
                return pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        return pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_index))

    def start(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def loop():
                while not self._stop.is_set():
                    try:
                        t = time.perf_counter()
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((t, float(sm), float(smax), pw, int(rs)))
                    except Exception:
                        pass
                    self._stop.wait(self.period_s)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = f"NVML, every {self.period_s * 1e3:.0f} ms"
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100", "-i", str(self.gpu_index)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi -lms 100"
            except Exception:
                self.proc = None
        time.sleep(0.05)

    def mark_start(self):
        self.t0 = time.perf_counter()
        self.d0 = _dt.datetime.now()

    def mark_end(self):
        self.t1 = time.perf_counter()
        self.d1 = _dt.datetime.now()

    def _summary(self, rows, inside):
        sm = [r[1] for r in rows]
        reasons = set()
        for r in rows:
            for bit, name in _NVML_REASONS.items():
                if r[4] & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max((r[2] for r in rows if r[2] is not None), default=None),
                "reasons": sorted(reasons), "samples": len(rows),
                "window": "timed region" if inside else "whole run (no sample fell inside the timed region)",
                "power_w_max": max((r[3] for r in rows if r[3] is not None), default=None),
                "source": self.source}

    def stop(self):
        if self.thread is not None:
            time.sleep(0.01)
            self._stop.set()
            self.thread.join(timeout=5)
            inside = [r for r in self.samples if self.t0 is not None and self.t0 <= r[0] <= self.t1]
            return self._summary(inside if inside else self.samples, bool(inside))
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"],
                    "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                continue
            num = lambda x: float(x) if x.replace(".", "").isdigit() else None
            bits = 0
            for bit, val in zip((0x8, 0x40, 0x20, 0x4), parts[6:10]):
                if val.lower().startswith("active"):
                    bits |= bit
            rows.append((ts, num(parts[2]), num(parts[3]), num(parts[4]), bits))
        inside = [r for r in rows if self.t0 is not None and self.d0 <= r[0] <= self.d1]
        sample = inside if inside else rows
        sample = [r for r in sample if r[1] is not None]
        return self._summary(sample, bool(inside))


# --------------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, world


def dist_init(backend: str, local: int):
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend=backend, timeout=_dt.timedelta(seconds=120))
    return dist


def reduce_max(value: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(useful_flops_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the work of every rank over the slowest rank's time."""
    return world * useful_flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


# --------------------------------------------------------------------- CPU oracle timing
def oracle_sample(w, bands, prefix_rows: int):
    """Time the fp64 oracle's forward + backward on a causal prefix of head 0
    of batch 0: query rows [0, prefix_rows) with that head's band.  Those rows'
    outputs equal the full-sequence ones (causal rows only look back).
    Returns (useful flops, seconds, threads, description)."""
    import oracle
    q, k, v, do = synth.make_inputs(1, 1, prefix_rows, w.d, seed=w.seed)
    f = lambda t: t.to(torch.float64).numpy()
    lo, hi = [bands[0][0]], [bands[1][0]]
    t0 = time.perf_counter()
    oracle.spa_fwd(f(q), f(k), f(v), w.scale, lo, hi)
    oracle.spa_bwd(f(q), f(k), f(v), f(do), w.scale, lo, hi)
    secs = time.perf_counter() - t0
    pairs = band_pairs_prefix(prefix_rows, lo[0], hi[0])
    desc = (f"oracle spa_fwd + spa_bwd (fp64, OpenMP) on head 0, query rows [0, {prefix_rows}) "
            f"of the {w.name} workload (band [{lo[0]}, {hi[0]}), d={w.d}); {pairs} pairs")
    return 14 * w.d * pairs, secs, oracle.num_threads(), desc


def oracle_union_sample(w, bands, window: int, prefix_rows: int):
    """The union oracle's forward + backward on a causal prefix of head 1 of
    batch 0 (its band and the window do not touch there).  Returns (useful
    flops, seconds, threads, description)."""
    import oracle
    q, k, v, do = synth.make_inputs(1, 1, prefix_rows, w.d, seed=w.seed)
    f = lambda t: t.to(torch.float64).numpy()
    h = 1 if len(bands[0]) > 1 else 0
    lo, hi = [bands[0][h]], [bands[1][h]]
    t0 = time.perf_counter()
    oracle.union_fwd(f(q), f(k), f(v), w.scale, window, lo, hi)
    oracle.union_bwd(f(q), f(k), f(v), f(do), w.scale, window, lo, hi)
    secs = time.perf_counter() - t0
    pairs = union_pairs(prefix_rows, window, (lo, hi))
    desc = (f"oracle union_fwd + union_bwd (fp64, OpenMP) on head {h}, query rows [0, {prefix_rows}) of the "
            f"{w.name} workload (band [{lo[0]}, {hi[0]}), window {window}, d={w.d}); {pairs} pairs")
    return 14 * w.d * pairs, secs, oracle.num_threads(), desc


def calibrate_union_prefix(w, bands, window: int, target_s: float, start: int = 1024):
    P = min(start, w.N)
    while True:
        fl, secs, cores, desc = oracle_union_sample(w, bands, window, P)
        if secs >= target_s / 2 or P >= w.N:
            return P, fl, secs, cores, desc
        P = min(2 * P, w.N)


def calibrate_prefix(w, bands, target_s: float, start: int = 256):
    """Double the prefix until one oracle run takes at least target_s / 2 (or
    the prefix covers the sequence).  Returns the last run:
    (prefix, flops, seconds, threads, description)."""
    P = min(start, w.N)
    while True:
        fl, secs, cores, desc = oracle_sample(w, bands, P)
        if secs >= target_s / 2 or P >= w.N:
            return P, fl, secs, cores, desc
        P = min(2 * P, w.N)


def run_reference(args):
    rank, local, world = dist_setup()
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    import oracle
    lo, hi = oracle.bands(w.N, w.H)
    bands = ([int(x) for x in lo], [int(x) for x in hi])
    budget = 150.0  # seconds for the whole --steps/--warmup run
    per_step = budget / max(args.steps + args.warmup, 1)
    P = calibrate_prefix(w, bands, min(per_step, 20.0), start=128)[0]
    for _ in range(args.warmup):
        oracle_sample(w, bands, P)
    total_flops, total_s = 0.0, 0.0
    for _ in range(args.steps):
        fl, s, cores, desc = oracle_sample(w, bands, P)
        total_flops += fl
        total_s += s
    value = total_flops / total_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": spa_config(w, w.B * workload_pairs(w.N, bands), world, False),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- decode step
DECODE_METRIC = "band-sparse decode step (one new token per sequence): GB/s of band K/V read"
DECODE_CONFIG = {"workload": "decode_b16_h32_n32768_d128", "B": 16, "H": 32, "N": 32768, "d": 128}


def decode_bytes(d, bands, positions):
    """Algorithmic bytes of one decode call: the band's keys and values read
    once per (b, h), q read, o and lse written."""
    total = 0
    for t in positions:
        for lo, hi in zip(*bands):
            jlo, jhi = max(0, t - hi + 1), t - lo
            total += 2 * max(0, jhi - jlo + 1) * d * 2 + d * 2 + d * 2 + 4
    return total


def run_decode(args):
    """One decode call per step on the B16 H32 N32768 d128 cache, every
    sequence at its last position (each head reads its full band)."""
    from head_partitioned_distance_b200 import spa

    rank, local, world = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); there is no CPU path")
    dist = dist_init("nccl", local) if world > 1 else None
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    B, H, N, d = (DECODE_CONFIG[x] for x in ("B", "H", "N", "d"))
    scale = d ** -0.5
    bands = spa.spa_band_bounds(N, H)
    # seeded synthetic inputs, generated on the device (the cache is 8.6 GB)
    gen = torch.Generator(device=device).manual_seed(5000 + 7919 * rank)
    kc = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    q = torch.randn((B, H, d), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    positions = [N - 1] * B
    pos = torch.tensor(positions, dtype=torch.int32, device=device)
    o = torch.empty((B, H, d), dtype=torch.bfloat16, device=device)
    lse = torch.empty((B, H), dtype=torch.float32, device=device)
    ws = torch.empty(spa.spa_attn_decode_workspace_bytes(B, H, N, d) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    step = lambda: spa.spa_attn_decode(q, kc, vc, pos, o, lse, ws, scale, stream=stream)
    nbytes = decode_bytes(d, bands, positions)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after warm-up")
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local] if visible else local, device)
    sampler.start()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.mark_start()
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_end()
    clocks = sampler.stop()
    max_ms = reduce_max(e0.elapsed_time(e1), device)
    value = world * nbytes * K / (max_ms * 1e-3) / 1e9
    # end to end: the new tokens' queries and positions from pinned host
    # memory, o and lse back, inside the timed region; as in the training
    # step, neighbouring calls' copies overlap on three streams with two
    # sets of device buffers (the cache is shared, read only)
    q_h, pos_h = q.cpu().pin_memory(), pos.cpu().pin_memory()
    o_h, lse_h = torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(lse.shape).pin_memory()
    sets = [dict(q=q, pos=pos, o=o, lse=lse, ws=ws)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    h2d_done, cmp_done, d2h_done = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))

    def e2e_run(steps):
        for s_ in range(steps):
            x = s_ % 2
            S = sets[x]
            if s_ >= 2:
                s_h2d.wait_event(cmp_done[x])
            with torch.cuda.stream(s_h2d):
                S["q"].copy_(q_h, non_blocking=True)
                S["pos"].copy_(pos_h, non_blocking=True)
                h2d_done[x].record(s_h2d)
            stream.wait_event(h2d_done[x])
            if s_ >= 2:
                stream.wait_event(d2h_done[x])
            spa.spa_attn_decode(S["q"], kc, vc, S["pos"], S["o"], S["lse"], S["ws"], scale, stream=stream)
            cmp_done[x].record(stream)
            s_d2h.wait_event(cmp_done[x])
            with torch.cuda.stream(s_d2h):
                o_h.copy_(S["o"], non_blocking=True)
                lse_h.copy_(S["lse"], non_blocking=True)
                d2h_done[x].record(s_d2h)

    E = max(8, min(200, K))
    e2e_run(4)
    torch.cuda.synchronize(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_h2d)
    e2e_run(E)
    f1.record(s_d2h)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(f0.elapsed_time(f1), device)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the timed region")
    if rank == 0:
        peaks, peak_src = load_peaks()
        per_gpu = value / world
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            # the oracle's forward rows on head 0's slice of the first
            # sequence: the decode of that (b, h) at several positions
            kf = kc[0, :1].unsqueeze(0).double().cpu().numpy()
            vf = vc[0, :1].unsqueeze(0).double().cpu().numpy()
            qf = np.zeros_like(kf)
            rows = list(range(N - 1, -1, -1))
            qf[0, 0, rows, :] = q[0, 0].double().cpu().numpy()
            lo0, hi0 = [bands[0][0]], [bands[1][0]]
            # repeat the N positions until about half the target CPU time
            reps, secs = 0, 0.0
            while secs < args.cpu_seconds / 2:
                t0 = time.perf_counter()
                oracle.spa_fwd_rows(qf, kf, vf, scale, rows, lo0, hi0)
                secs += time.perf_counter() - t0
                reps += 1
            cb = reps * decode_bytes(d, (lo0, hi0), rows)
            cpu = {"value": cb / secs / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                   "sample": f"oracle spa_fwd_rows (fp64) for all {N} decode positions of head 0 "
                             f"(band [{lo0[0]}, {hi0[0]})) of sequence 0, {reps} times", "seconds": secs}
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": max_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**DECODE_CONFIG, "positions": "N - 1 for every sequence",
                       "bands": "balanced distance partitioning", "bytes_per_call": nbytes,
                       "l2": f"no flush: the bands' K/V ({nbytes / 2**20:.0f} MiB) exceed L2",
                       "parallelism": f"{world} independent replicas"},
            "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": per_gpu / peaks["hbm_gbs"], "traffic": None,
                         "kernel": "spa_decode_chunk_kernel + spa_decode_merge_kernel",
                         "peak_source": f"{peak_src} (hbm_gbs)"},
            "cpu_baseline": cpu,
            "e2e": {"value": world * nbytes * E / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": q.numel() * 2 + B * 4, "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4,
                    "steps": E, "ms_per_step": e2e_ms / E,
                    "schedule": "H2D, decode and D2H on three streams with two device buffer sets"},
            "gpu_launches": 2 * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# --------------------------------------------------------------------- GPU arm
E2E_SCHEDULE = ("H2D, compute and D2H on three streams with two device buffer sets: each step's copies "
                "overlap its neighbours' compute and copies")


def pipelined_e2e(device, stream, host, dev0, out_names, compute, E, dist):
    """End-to-end time of E steps through the public API with host buffers.
    Every step copies its inputs (``host``: name -> CPU tensor, same names in
    ``dev0``) in from pinned host memory and its outputs (``out_names``) back.
    As a caller streaming batches would, the copies of neighbouring steps
    overlap the compute: H2D, compute and D2H run on three streams over two
    device buffer sets, so PCIe carries both directions at once.  ``compute``
    launches one step on a buffer set (a dict like ``dev0``) on ``stream``.
    Returns (max-over-ranks ms for the E steps, H2D bytes, D2H bytes per step)."""
    pin = {n: t.pin_memory() for n, t in host.items()}
    out_h = {n: torch.empty(dev0[n].shape, dtype=dev0[n].dtype).pin_memory() for n in out_names}
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in out_h.values())
    sets = [dev0, {n: torch.empty_like(t) for n, t in dev0.items()}]
    s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    h2d_done, cmp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(steps):
        for s_ in range(steps):
            x = s_ % 2
            S = sets[x]
            if s_ >= 2:
                s_h2d.wait_event(cmp_done[x])  # step s - 2 has read this set's inputs
            with torch.cuda.stream(s_h2d):
                for n in pin:
                    S[n].copy_(pin[n], non_blocking=True)
                h2d_done[x].record(s_h2d)
            stream.wait_event(h2d_done[x])
            if s_ >= 2:
                stream.wait_event(d2h_done[x])  # step s - 2's outputs have left this set
            compute(S)
            cmp_done[x].record(stream)
            s_d2h.wait_event(cmp_done[x])
            with torch.cuda.stream(s_d2h):
                for n in out_h:
                    out_h[n].copy_(S[n], non_blocking=True)
                d2h_done[x].record(s_d2h)

    run(2)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    stream.wait_event(e0)
    run(E)
    s_d2h.wait_event(cmp_done[(E - 1) % 2])
    e1.record(s_d2h)
    torch.cuda.synchronize(device)
    return reduce_max(e0.elapsed_time(e1), device), h2d, d2h


def flush_needed(w) -> bool:
    """Inputs smaller than L2 are flushed out of it before every timed step."""
    return w.B * w.H * w.N * w.d * 2 < L2_BYTES


def spa_config(w, pairs: int, world: int, full_bands: bool):
    """The "config" object of the training-step line (both arms print it)."""
    B, H, N, d = w.B, w.H, w.N, w.d
    return {"workload": w.name, "B": B, "H": H, "N": N, "d": d,
            "bands": ("full: [0, N) on every head (dense causal per head)" if full_bands
                      else "balanced distance partitioning"),
            "pairs_per_rank": pairs,
            "useful_flops_per_rank_step": 14 * d * pairs,
            "l2": (f"flushed before every step (a {2 * L2_BYTES / 2**20:.0f} MiB write, then a "
                   f"{HOST_LEAD_CYCLES}-cycle device wait; neither timed)") if flush_needed(w) else
                  ("no flush: q, k, v, dout are each larger than L2 "
                   f"({B * H * N * d * 2 / 2**20:.0f} MiB bf16)"),
            "parallelism": f"{world} independent replicas (one batch each)"}


SWEEP = [("b1_h4_n256_d64", 50, False), ("b1_h8_n1024_d64", 50, False), ("b1_h8_n1000_d64", 50, False),
         ("b1_h8_n1001_d64", 50, False), ("b8_h16_n4096_d128", 20, False), ("b4_h32_n8192_d128", 20, False),
         ("b1_h32_n32768_d128", 10, False), ("b1_h32_n30001_d128", 10, False), ("b4_h32_n8192_d128", 3, True),
         ("b1_h32_n32768_d128", 3, True)]


def backward_call(spa, mode: str, B: int, H: int, N: int, d: int, device, bands=None):
    """(the public backward entry of a mode, a workspace for it)."""
    lo, hi = (None, None) if bands is None else bands
    if mode == "fused":
        return spa.spa_attn_bwd_fused, torch.empty(spa.spa_attn_bwd_fused_workspace_bytes(B, H, N, d) // 4,
                                                   dtype=torch.float32, device=device)
    if mode == "stored":
        return spa.spa_attn_bwd_stored, torch.empty(spa.spa_attn_bwd_stored_workspace_bytes(B, H, N, d, lo, hi),
                                                    dtype=torch.uint8, device=device)
    return spa.spa_attn_bwd, torch.empty(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32,
                                         device=device)


def sweep_workloads(spa, device, stream, peaks, mode: str, warmup: int = 3):
    """Every workload of the scope table, a few steps each, after the headline
    measurement: ms per step, useful TFLOP/s, % of the bf16 peak, tokens/s and
    the step's roofline fraction, plus the same kernels with full bands (dense
    causal attention on every head) at two sizes.  The band workloads run with
    the headline's backward and, when that is not the two-pass one, with the
    two-pass backward too (key "<workload>/two-pass"); the full-band runs use
    the two-pass backward.  Inputs are drawn on the device with each
    workload's recipe; workloads smaller than L2 are flushed out of it before
    every step (untimed); each step is timed with CUDA events on the launching
    stream and the steps' times are summed."""
    out = {}
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    runs = []
    for name, K, full in SWEEP:
        if full:
            runs.append((name, K, full, "two-pass"))
        else:
            runs.append((name, K, full, mode))
            if mode != "two-pass":
                runs.append((name, K, full, "two-pass"))
    for name, K, full, bmode in runs:
        w = synth.WORKLOADS[name]
        B, H, N, d = w.B, w.H, w.N, w.d
        bands = ([0] * H, [N] * H) if full else spa.spa_band_bounds(N, H)
        lo_hi = {"lo": bands[0], "hi": bands[1]} if full else {}
        q, k, v, do = synth.make_inputs(B, H, N, d, w.seed, w.qkv_mult, w.rms_qk, w.do_mult, device=device)
        o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
        lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
        bwd, ws = backward_call(spa, bmode, B, H, N, d, device, bands if full else None)

        def step():
            spa.spa_attn_fwd(q, k, v, o, lse, w.scale, stream=stream, **lo_hi)
            bwd(q, k, v, o, do, lse, dq, dk, dv, ws, w.scale, stream=stream, **lo_hi)

        for _ in range(warmup):
            step()
        small = flush_needed(w)
        ms = 0.0
        for _ in range(K):
            if small:
                flush.fill_(1.0)
                torch.cuda._sleep(HOST_LEAD_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            e1.synchronize()
            ms += e0.elapsed_time(e1)
        if spa.spa_device_status(stream) != spa.SPA_OK:
            raise SystemExit(f"device status not OK in the sweep ({name})")
        pairs = B * workload_pairs(N, bands)
        flops, nbytes = step_work(w, pairs, active_rows(w, bands))
        step_ms = ms / K
        sr = step_roofline_report(flops, nbytes, step_ms, peaks)
        key = name + ("/full-bands" if full else "") + ("/two-pass" if bmode != mode and not full else "")
        out[key] = {
            "backward": bmode, "steps": K, "ms_per_step": step_ms, "useful_tflops": flops / (step_ms * 1e-3) / 1e12,
            "pct_of_bf16_peak": 100.0 * flops / (step_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "tokens_per_s": B * N / (step_ms * 1e-3), "step_bound": sr["bound"],
            "pct_of_step_roofline": 100.0 * sr["frac"], "pairs": pairs,
            "l2": "flushed before every step" if small else "inputs larger than L2"}
        del q, k, v, do, o, dq, dk, dv, lse, ws
        torch.cuda.empty_cache()
    return out


BACKWARD_DESCRIPTION = {
    "two-pass": "two passes (spa_attn_bwd: dQ pass forming D, dK/dV pass)",
    "fused": "one pass over key tiles (spa_attn_bwd_fused: prep, pass, dq convert)",
    "stored": "dS stored (spa_attn_bwd_stored: D, dK/dV pass writing each tile pair's dS^T, dQ from the tiles)",
}


def run_spa(args):
    from head_partitioned_distance_b200 import spa

    rank, local, world = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); there is no CPU path")
    dist = dist_init("nccl", local) if world > 1 else None
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[args.workload]
    B, H, N, d = w.B, w.H, w.N, w.d
    if args.full_bands:
        # every head's band is [0, N): dense causal attention on every head,
        # through the same kernels (the explicit-band entry points)
        bands = ([0] * H, [N] * H)
        lo_hi = {"lo": bands[0], "hi": bands[1]}
    else:
        bands = spa.spa_band_bounds(N, H)
        lo_hi = {}
    pairs = B * workload_pairs(N, bands)
    useful = 14 * d * pairs

    # independent batch per rank (weak scaling)
    q, k, v, do = synth.make_inputs(B, H, N, d, w.seed + 7919 * rank, w.qkv_mult, w.rms_qk, w.do_mult)
    host = {"q": q, "k": k, "v": v, "do": do}
    qd, kd, vd, dod = (t.to(device) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    ws = torch.empty(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    scale = w.scale
    # inputs smaller than L2 are flushed out of it before every timed step (a
    # write of a buffer twice its size, outside the timed spans)
    flush = None
    if flush_needed(w):
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    mode = args.bwd
    kernels = KERNELS_OF[mode]
    bwd_call, ws = backward_call(spa, mode, B, H, N, d, device, bands if args.full_bands else None)

    def step(ev=None):
        spa.spa_attn_fwd(qd, kd, vd, o, lse, scale, stream=stream, **lo_hi)
        if ev is not None:
            ev[1].record(stream)
        if mode in ("fused", "stored"):
            # the three launches of the backward, an event after each
            for i, st in enumerate((1, 2, 4)):
                bwd_call(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, scale, stream=stream, steps=st, **lo_hi)
                if ev is not None:
                    ev[2 + i].record(stream)
            return
        spa.spa_attn_bwd_dq_delta(qd, kd, vd, o, dod, lse, ws, dq, scale, stream=stream, **lo_hi)
        if ev is not None:
            ev[2].record(stream)
        spa.spa_attn_bwd_dkdv(qd, kd, vd, dod, lse, ws, dk, dv, scale, stream=stream, **lo_hi)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after warm-up")

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local] if visible else local, device)
    sampler.start()
    K = args.steps
    # per step: its start, then the end of each kernel
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(kernels) + 1)] for _ in range(K)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.mark_start()
    for s in range(K):
        if flush is not None:
            flush.fill_(float(s))
            # a short device-side wait, untimed, lets the host queue the
            # step's three calls before the GPU reaches them, so that the
            # timed spans hold device time and not the host's call overhead
            torch.cuda._sleep(HOST_LEAD_CYCLES)
        evs[s][0].record(stream)
        step(evs[s])
    torch.cuda.synchronize(device)
    sampler.mark_end()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the timed region")
    if flush is None:
        elapsed_ms = evs[0][0].elapsed_time(evs[-1][-1])
    else:
        elapsed_ms = sum(e[0].elapsed_time(e[-1]) for e in evs)
    per_kernel_ms = {name: 0.0 for name in kernels}
    for e in evs:
        for i, name in enumerate(kernels):
            per_kernel_ms[name] += e[i].elapsed_time(e[i + 1])
    max_ms = reduce_max(elapsed_ms, device)
    value = aggregate(useful, K, world, max_ms)

    # ------------------------------------------------ end to end, host buffers
    E = max(4, min(16, K))
    dev0 = dict(q=qd, k=kd, v=vd, do=dod, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)

    def compute(S):
        spa.spa_attn_fwd(S["q"], S["k"], S["v"], S["o"], S["lse"], scale, stream=stream, **lo_hi)
        bwd_call(S["q"], S["k"], S["v"], S["o"], S["do"], S["lse"], S["dq"], S["dk"], S["dv"], S["ws"], scale,
                 stream=stream, **lo_hi)

    e2e_ms, h2d, d2h = pipelined_e2e(device, stream, host, dev0, ("o", "lse", "dq", "dk", "dv"), compute, E,
                                     dist)
    e2e_value = aggregate(useful, E, world, e2e_ms)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the end-to-end region")

    if rank == 0:
        peaks, peak_src = load_peaks()
        act = active_rows(w, bands)
        work = kernel_work(w, pairs, act, stored_tiles(spa, w, bands) if mode == "stored" else 0)
        kern = {name: kernel_report(*work[name], per_kernel_ms[name] / K, per_kernel_ms[name] / elapsed_ms,
                                    peaks) for name in kernels}
        # the whole step against its attainable roofline: the slower of the
        # useful FLOPs at the bf16 peak and the bytes any forward + backward
        # must move at the HBM peak
        step_flops, step_bytes = step_work(w, pairs, act)
        step_roofline = step_roofline_report(step_flops, step_bytes, max_ms / K, peaks)
        dom = max(kernels, key=lambda n: per_kernel_ms[n])
        dk_ = kern[dom]
        roofline = {"bound": dk_["bound"], "achieved": dk_["achieved"], "peak": dk_["peak"],
                    "unit": dk_["unit"], "frac": dk_["frac"],
                    "traffic": ncu_traffic(dom, w.name + ("/full-bands" if args.full_bands else "")),
                    "kernel": dom,
                    "algorithmic_per_launch": dk_["algorithmic_per_launch"],
                    "peak_source": f"{peak_src} ({'bf16_tflops burst' if dk_['bound'] == 'tensor' else 'hbm_gbs'})"}
        per_workload = None
        if world == 1 and not args.no_sweep:
            per_workload = sweep_workloads(spa, device, stream, peaks, mode)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            P, fl, secs, cores, desc = calibrate_prefix(w, bands, args.cpu_seconds, start=512)
            cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": desc, "seconds": secs}
        per_gpu = value / world
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": max_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "pct_of_bf16_peak": 100.0 * per_gpu / peaks["bf16_tflops"],
            # the metric's literal wording: 10 d per pair over the fwd+bwd time
            # (the headline counts 14 d: the forward's 4 d and the backward's 10 d)
            "value_literal_10d": value * 10.0 / 14.0,
            "pct_of_bf16_peak_literal_10d": 100.0 * per_gpu * 10.0 / 14.0 / peaks["bf16_tflops"],
            "pct_of_bf16_peak_sustained": 100.0 * per_gpu / peaks["bf16_tflops_sustained"],
            "peaks": {**peaks, "source": peak_src},
            "tokens_per_s": world * B * N * K / (max_ms * 1e-3),
            "config": spa_config(w, pairs, world, args.full_bands),
            "roofline": roofline,
            "step_roofline": step_roofline,
            "kernels": kern,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": E, "ms_per_step": e2e_ms / E,
                    "schedule": E2E_SCHEDULE},
            "per_workload": per_workload,
            "gpu_launches": len(kernels) * K,
            "backward": BACKWARD_DESCRIPTION[mode],
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# one union step, launch by launch: (name, what it runs)
UNION_LAUNCHES = ("fwd part 1", "fwd part 2 (merging)", "dq+D part 1", "dk/dv part 1", "dq part 2 (adding)",
                  "dk/dv part 2 (adding)")
UNION_KERNEL_OF = {"fwd part 1": "spa_fwd_kernel", "fwd part 2 (merging)": "spa_fwd_kernel",
                   "dq+D part 1": "spa_bwd_dq_kernel",
                   "dk/dv part 1": "spa_bwd_dkdv_kernel", "dq part 2 (adding)": "spa_bwd_dq_kernel",
                   "dk/dv part 2 (adding)": "spa_bwd_dkdv_kernel"}


def run_union(args):
    """Band plus a local window [0, W) shared by every head (spa_attn_fwd_union
    + spa_attn_bwd_union) on the same workload; useful FLOPs over the union's
    pairs."""
    from head_partitioned_distance_b200 import spa

    rank, local, world = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); there is no CPU path")
    dist = dist_init("nccl", local) if world > 1 else None
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[args.workload]
    B, H, N, d = w.B, w.H, w.N, w.d
    W = args.union
    bands = spa.spa_band_bounds(N, H)
    a1, b1, a2, b2 = spa.spa_union_parts(N, H, W)
    pairs = B * union_pairs(N, W, bands)
    pairs1 = B * workload_pairs(N, (a1, b1))
    pairs2 = B * workload_pairs(N, (a2, b2))
    assert pairs1 + pairs2 == pairs
    useful = 14 * d * pairs

    q, k, v, do = synth.make_inputs(B, H, N, d, w.seed + 7919 * rank, w.qkv_mult, w.rms_qk, w.do_mult)
    host = {"q": q, "k": k, "v": v, "do": do}
    qd, kd, vd, dod = (t.to(device) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    ws = torch.empty(spa.spa_attn_union_workspace_bytes(B, H, N, d) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    scale = w.scale

    def step(S):
        spa.spa_attn_fwd_union(S["q"], S["k"], S["v"], S["o"], S["lse"], scale, W, stream=stream)
        spa.spa_attn_bwd_union(S["q"], S["k"], S["v"], S["o"], S["do"], S["lse"], S["dq"], S["dk"], S["dv"],
                               S["ws"], scale, W, stream=stream)

    dev0 = dict(q=qd, k=kd, v=vd, do=dod, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)
    for _ in range(args.warmup):
        step(dev0)
    torch.cuda.synchronize(device)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after warm-up")

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local] if visible else local, device)
    sampler.start()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.mark_start()
    t0.record(stream)
    for _ in range(K):
        step(dev0)
    t1.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_end()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the timed region")
    max_ms = reduce_max(t0.elapsed_time(t1), device)
    value = aggregate(useful, K, world, max_ms)

    # the same launches one public call at a time, with an event after each:
    # per-launch durations for the shares and the roofline
    wsb = torch.empty(spa.spa_attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device=device)
    calls = [
        lambda: spa.spa_attn_fwd(qd, kd, vd, o, lse, scale, a1, b1, stream=stream),
        lambda: spa.spa_attn_fwd_merge(qd, kd, vd, o, lse, scale, a2, b2, stream=stream),
        lambda: spa.spa_attn_bwd_dq_delta(qd, kd, vd, o, dod, lse, wsb, dq, scale, a1, b1, stream=stream),
        lambda: spa.spa_attn_bwd_dkdv(qd, kd, vd, dod, lse, wsb, dk, dv, scale, a1, b1, stream=stream),
        lambda: spa.spa_attn_bwd_dq_add(qd, kd, vd, dod, lse, wsb, dq, scale, a2, b2, stream=stream),
        lambda: spa.spa_attn_bwd_dkdv_add(qd, kd, vd, dod, lse, wsb, dk, dv, scale, a2, b2, stream=stream),
    ]
    Kd = max(3, min(K, 20))
    for _ in range(2):
        for c in calls:
            c()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(Kd)]
    for s_ in range(Kd):
        evs[s_][0].record(stream)
        for i, c in enumerate(calls):
            c()
            evs[s_][i + 1].record(stream)
    torch.cuda.synchronize(device)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the launch-by-launch pass")
    launch_ms = {n: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / Kd for i, n in enumerate(UNION_LAUNCHES)}
    step_ms = sum(launch_ms.values())

    E = max(4, min(16, K))
    e2e_ms, h2d, d2h = pipelined_e2e(device, stream, host, dev0, ("o", "lse", "dq", "dk", "dv"), step, E, dist)
    e2e_value = aggregate(useful, E, world, e2e_ms)
    if spa.spa_device_status(stream) != spa.SPA_OK:
        raise SystemExit("device status not OK after the end-to-end region")

    if rank == 0:
        peaks, peak_src = load_peaks()
        kern = {}
        for name in sorted(set(UNION_KERNEL_OF.values())):
            ms = sum(launch_ms[n] for n in UNION_LAUNCHES if UNION_KERNEL_OF[n] == name)
            kern[name] = {"ms_per_step": ms, "share": ms / step_ms,
                          "launches_per_step": sum(1 for n in UNION_LAUNCHES if UNION_KERNEL_OF[n] == name)}
        # dominant kernel: the dK/dV pass, over both parts' pairs
        dk_ms = kern["spa_bwd_dkdv_kernel"]["ms_per_step"]
        achieved = 8 * d * pairs / (dk_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"], "traffic": None, "kernel": "spa_bwd_dkdv_kernel",
                    "per": "both launches of one step (parts 1 and 2): 8 d x union pairs over their summed time",
                    "peak_source": f"{peak_src} (bf16_tflops burst)"}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            P, fl, secs, cores, desc = calibrate_union_prefix(w, bands, W, args.cpu_seconds)
            cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": desc, "seconds": secs}
        line = {
            "metric": METRIC + " (band plus shared local window)", "value": value, "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": max_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "pct_of_bf16_peak": 100.0 * value / world / peaks["bf16_tflops"],
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d,
                       "bands": "balanced distance partitioning", "window": W,
                       "parts": "two disjoint distance intervals per head (spa_union_parts)",
                       "pairs_per_rank": pairs, "useful_flops_per_rank_step": useful,
                       "l2": "no flush: q, k, v, dout are each larger than L2",
                       "parallelism": f"{world} independent replicas (one batch each)"},
            "roofline": roofline,
            "kernels": kern,
            "launches_ms": launch_ms,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": E, "ms_per_step": e2e_ms / E, "schedule": E2E_SCHEDULE},
            "gpu_launches": len(UNION_LAUNCHES) * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def free_port() -> int:
    import socket
    s_ = socket.socket()
    s_.bind(("127.0.0.1", 0))
    port = s_.getsockname()[1]
    s_.close()
    return port


def relaunch(nproc: int, argv) -> int:
    """`--gpus N` without a torchrun world: start N ranks on this node with
    torch.distributed.run (rendezvous on 127.0.0.1) running this same
    command line, and return their exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_dry(args):
    """The launch and reporting path without any GPU work: every rank joins a
    gloo group, takes part in the barrier and the max over ranks of a
    (host-timed, trivial) step time, and rank 0 prints the line.  Lets a CPU
    machine check what --gpus N does."""
    rank, local, world = dist_setup()
    dist = dist_init("gloo", local) if world > 1 else None
    t0 = time.perf_counter()
    x = torch.ones(64)
    for _ in range(args.steps):
        x = x * 1.0
    ms = (time.perf_counter() - t0) * 1e3
    if dist:
        dist.barrier()
    max_ms = reduce_max(ms, torch.device("cpu"))
    if rank == 0:
        print(json.dumps({"dry_run": True, "metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": max_ms / max(args.steps, 1),
                          "ranks_reporting": world, "config": {"workload": args.workload}}), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["spa", "reference"], default="spa")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the short run of every other workload (and of the full bands) after the headline")
    ap.add_argument("--union", type=int, default=0, metavar="W",
                    help="time band plus a local window [0, W) shared by every head instead")
    ap.add_argument("--full-bands", action="store_true",
                    help="run every head with the full band [0, N) (dense causal per head) through the same "
                         "kernels, to show the work the bands save")
    ap.add_argument("--bwd", choices=["stored", "two-pass", "fused"], default="stored",
                    help="backward of the timed step: the one that stores dS (spa_attn_bwd_stored, "
                         "deterministic; the default), the two-pass one (spa_attn_bwd, deterministic) or the "
                         "one-pass one (spa_attn_bwd_fused)")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode step (one new token per sequence) instead of fwd+bwd")
    ap.add_argument("--ncu-summary", metavar="CSV",
                    help="print the markdown summary of one launch from `ncu -i REP --page raw --csv` output "
                         "(with --ncu-kernel, --ncu-command; --workload names the workload captured)")
    ap.add_argument("--ncu-launch-list", metavar="CSV",
                    help="print the markdown launch list from `ncu --metrics gpu__time_duration.sum --csv` output "
                         "(with --ncu-command; --bench-json adds the bench line's event shares)")
    ap.add_argument("--bench-json", default="")
    ap.add_argument("--ncu-kernel", default="")
    ap.add_argument("--ncu-command", default="")
    ap.add_argument("--ncu-note", default="")
    ap.add_argument("--src-sha", default="", help="kernel sources the capture ran on (default: the current ones)")
    ap.add_argument("--dry-run", action="store_true",
                    help="run the launch and reporting path (ranks, barrier, max over ranks) with no GPU work")
    args = ap.parse_args(argv)
    if args.ncu_launch_list:
        print(ncu_launch_list(args.ncu_launch_list, args.workload, args.ncu_command, args.bench_json, args.ncu_note),
              end="")
        return 0
    if args.ncu_summary:
        print(ncu_summary(args.ncu_summary, args.ncu_kernel, args.workload, args.ncu_command,
                          args.src_sha or kernel_src_sha(), args.ncu_note), end="")
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return relaunch(args.gpus, argv)  # one rank per GPU, this node
    if world_env is not None and int(world_env) != args.gpus:
        ap.error(f"--gpus {args.gpus} but this process is one of a world of {world_env} ranks")
    if args.dry_run:
        return run_dry(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.decode:
        return run_decode(args)
    if args.union:
        return run_union(args)
    return run_spa(args)


if __name__ == "__main__":
    sys.exit(main())
