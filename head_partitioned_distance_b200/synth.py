"""Seeded synthetic inputs for SPAttention band-sparse attention.

This module only draws and shapes random tensors.  It holds none of the
method's arithmetic (no bands, no softmax, no gradients), so both the CUDA
path and the CPU oracle can take their inputs from it.

Recipe (the pages evaluate this path on no dataset; every input is synthetic):

* ``torch.Generator().manual_seed(seed)`` on the CPU; draws in the order Q, K,
  V, dO, each ``randn`` in fp32 of shape [B, H, N, d];
* per-workload transforms in fp32 (a multiplier on Q/K/V, RMS normalisation of
  Q and K rows over d -- x / sqrt(mean(x^2)) with no epsilon and no gain --, a
  multiplier on dO);
* a final cast to bf16.  Those bf16 bytes are what the GPU and the oracle see.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    seed: int
    qkv_mult: float = 1.0
    rms_qk: bool = False
    do_mult: float = 1.0
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> str:
        return f"B{self.B} H{self.H} N{self.N} d{self.d}"


# The five training-shaped workloads of this path, plus their ragged variants.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("b1_h4_n256_d64", 1, 4, 256, 64, 1000,
                 note="small case; bands of width 64"),
        Workload("b1_h8_n1024_d64", 1, 8, 1024, 64, 1001, qkv_mult=0.5,
                 note="Figure-1 layout of the paper: bands of width 128"),
        Workload("b1_h8_n1000_d64", 1, 8, 1000, 64, 1001, qkv_mult=0.5,
                 note="N not a multiple of the tile size; bands of width 125"),
        Workload("b1_h8_n1001_d64", 1, 8, 1001, 64, 1001, qkv_mult=0.5,
                 note="mixed band widths 125/126"),
        Workload("b8_h16_n4096_d128", 8, 16, 4096, 128, 1002, rms_qk=True, do_mult=1e-2,
                 note="training-shaped; RMS-normalised Q/K rows; dO scaled by 1e-2"),
        Workload("b4_h32_n8192_d128", 4, 32, 8192, 128, 1003,
                 note="7B-like attention layer"),
        Workload("b1_h32_n32768_d128", 1, 32, 32768, 128, 1004,
                 note="long context; bands of width 1024"),
        Workload("b1_h32_n30001_d128", 1, 32, 30001, 128, 1004,
                 note="ragged long context; band widths 937/938, tail tile partly filled"),
    ]
}


def _rms_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True))


def make_inputs(B: int, H: int, N: int, d: int, seed: int, qkv_mult: float = 1.0,
                rms_qk: bool = False, do_mult: float = 1.0, device=None):
    """Return bf16 tensors (q, k, v, dout), each [B, H, N, d], on the CPU (the
    values the oracle and the parity tests use) or, with ``device``, drawn by
    that device's generator with the same recipe (other values, same
    distribution; for timing runs)."""
    g = torch.Generator(device=device or "cpu").manual_seed(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    k = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    v = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    dout = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if rms_qk:
        q = _rms_rows(q)
        k = _rms_rows(k)
    if qkv_mult != 1.0:
        q, k, v = q * qkv_mult, k * qkv_mult, v * qkv_mult
    if do_mult != 1.0:
        dout = dout * do_mult
    return tuple(t.to(torch.bfloat16) for t in (q, k, v, dout))


def workload_inputs(w: Workload):
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.qkv_mult, w.rms_qk, w.do_mult)


def sample_rows(B: int, H: int, N: int, count: int, seed: int, per_head=()):
    """Flat row ids (b*H + h)*N + i, sorted and unique: each head's first and
    last row, the rows ``per_head[h]`` that the caller names for head h, and
    ``count`` random ones."""
    g = torch.Generator().manual_seed(seed)
    rows = set()
    for b in range(B):
        for h in range(H):
            base = (b * H + h) * N
            extra = list(per_head[h]) if h < len(per_head) else []
            for i in [0, N - 1] + extra:
                if 0 <= i < N:
                    rows.add(base + i)
    if count > 0:
        rows.update(torch.randint(0, B * H * N, (count,), generator=g).tolist())
    return sorted(rows)
