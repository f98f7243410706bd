"""Seeded synthetic inputs for attention workloads.

This module only draws random numbers and names workloads; it holds none of
the attention arithmetic.  Both the CUDA path's tests/benchmark and the CPU
oracle's tests take their inputs from here, so both sides see the same values.

Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws Q, K, V and dO,
in that order, as float32 standard normals of shape [B, H, N, d]; each is then
rounded to the workload's dtype (bf16 or fp32).  The oracle is fed exactly
those rounded values, widened to float64.

The workload shapes follow the GPT-2-style model table of the CS336 A2 Systems
handout (section 2.1.2, Table 1: small/medium/large/xl/10B with head dim
d_model / num_heads) and the sequence-length x head-dim sweep of its
flash_benchmarking problem (section 4.2.2: batch 1, causal, powers of two).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import torch

DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32, "fp16": torch.float16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "bf16" or "fp32"
    seed: int
    causal: bool = True

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def heads(self) -> int:
        return self.B * self.H


# Fixed workloads: the fp32 small case and the model-table head shapes.
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("fp32-b2h4-n128-d64", 2, 4, 128, 64, "fp32", 0),
    Workload("gpt2-small-b4h12-n512-d64", 4, 12, 512, 64, "bf16", 0),
    Workload("gpt2-medium-b4h16-n1024-d64", 4, 16, 1024, 64, "bf16", 0),
    Workload("gpt2-large-b4h20-n1024-d64", 4, 20, 1024, 64, "bf16", 0),
    Workload("gpt2-xl-b4h32-n2048-d80", 4, 32, 2048, 80, "bf16", 0),
    Workload("10b-b1h36-n4096-d128", 1, 36, 4096, 128, "bf16", 0),
]}

SWEEP_N = [128 << i for i in range(9)]          # 128 ... 32768
SWEEP_D = [16, 32, 64, 128]


def sweep_workload(N: int, d: int, dtype: str) -> Workload:
    """One point of the causal B=1, H=16 sequence-length x head-dim sweep."""
    return Workload(f"sweep-b1h16-n{N}-d{d}-{dtype}", 1, 16, N, d, dtype, 1000 + N + d)


def workload_by_name(name: str) -> Workload:
    """A fixed workload, or a sweep point named as sweep_workload names it
    ("sweep-b1h16-n<N>-d<d>-<dtype>")."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    parts = name.split("-")
    if len(parts) == 5 and parts[0] == "sweep" and parts[1] == "b1h16" and parts[4] in DTYPES:
        w = sweep_workload(int(parts[2][1:]), int(parts[3][1:]), parts[4])
        if w.name == name:
            return w
    raise KeyError(f"unknown workload {name!r}")


def sweep_workloads() -> List[Workload]:
    return [sweep_workload(N, d, dt) for dt in ("bf16", "fp32") for d in SWEEP_D for N in SWEEP_N]


def make_inputs(B: int, H: int, N: int, d: int, dtype: str, seed: int,
                with_grad_out: bool = True) -> Dict[str, torch.Tensor]:
    """Q, K, V (and dO) on the CPU, contiguous [B, H, N, d] in ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    names = ["q", "k", "v"] + (["do"] if with_grad_out else [])
    out = {}
    for nm in names:
        x = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
        out[nm] = x.to(DTYPES[dtype]).contiguous()
    return out


def workload_inputs(w: Workload, with_grad_out: bool = True) -> Dict[str, torch.Tensor]:
    return make_inputs(w.B, w.H, w.N, w.d, w.dtype, w.seed, with_grad_out)


def sample_rows(n: int, count: int, seed: int) -> List[int]:
    """Seeded distinct row indices in [0, n), always including 0 and n-1."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    count = min(count, n)
    picks = set([0, n - 1])
    perm = torch.randperm(n, generator=g).tolist()
    for r in perm:
        if len(picks) >= count:
            break
        picks.add(r)
    return sorted(picks)
