"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same inputs, compare element by element."""
from __future__ import annotations

import math

import numpy as np
import torch

# Per-element bound |gpu - ref| <= ATOL + RTOL * |ref|.
# fp16 inputs take the bf16 bound: both are 16-bit inputs with fp32
# accumulation and P, dS rounded to the input type.
TOL = {"bf16": (1e-2, 1e-2), "fp16": (1e-2, 1e-2), "fp32": (2e-3, 2e-3)}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, name: str) -> float:
    """Per-element tolerance check; returns the largest absolute error."""
    atol, rtol = TOL[dtype]
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values in the CUDA result"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{name}: {int(bad.sum())} of {err.size} elements out of tolerance "
            f"(atol={atol}, rtol={rtol}); worst at {idx}: got {got[idx]!r} ref {ref[idx]!r}; "
            f"max abs err {err.max():.3e}")
    return float(err.max()) if err.size else 0.0


def gpu_fwd_bwd(inp, causal: bool, scale: float, do_backward: bool = True):
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa2.forward(q, k, v, causal=causal, scale=scale)
    out = {"o": o, "lse": lse}
    if do_backward:
        do = inp["do"].to(dev)
        dq, dk, dv = fa2.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
