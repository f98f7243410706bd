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


def gpu_fwd_bwd(inp, causal: bool, scale: float, do_backward: bool = True,
                mode: str = "default"):
    """Forward and backward on cuda:0 through the binding; ``mode`` is the
    backward's form ("default", "two-pass" or "one-pass")."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa2.forward(q, k, v, causal=causal, scale=scale)
    out = {"o": o, "lse": lse}
    if do_backward:
        do = inp["do"].to(dev)
        dq, dk, dv = fa2.backward(q, k, v, o, lse, do, causal=causal, scale=scale,
                                  mode=mode)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def grouped_reference(oracle_mod, q, k, v, do, causal: bool, scale: float):
    """Oracle results for H query heads sharing H_kv key/value heads (query head
    h reads key/value head h // (H // H_kv)) with query length N and key length
    Nk: the oracle runs once per query head on that head's shared K and V, and
    dK, dV of a key/value head are the sums of the per-query-head gradients over
    the heads sharing it (the chain rule through the broadcast of K and V).
    Tensors are [B, H, N, d] and [B, H_kv, Nk, d]; results are float64 numpy."""
    B, H, N, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    grp = H // H_kv
    ref = {n: np.zeros(s) for n, s in (("o", (B, H, N, d)), ("lse", (B, H, N)), ("dq", (B, H, N, d)),
                                         ("dk", (B, H_kv, Nk, d)), ("dv", (B, H_kv, Nk, d)))}
    for b in range(B):
        for h in range(H):
            hk = h // grp
            qh, kh, vh, doh = (to64(t) for t in (q[b, h], k[b, hk], v[b, hk], do[b, h]))
            o, lse = oracle_mod.forward(qh, kh, vh, causal, scale)
            dq, dk, dv = oracle_mod.backward(qh, kh, vh, doh, causal, scale)
            ref["o"][b, h], ref["lse"][b, h], ref["dq"][b, h] = o, lse, dq
            ref["dk"][b, hk] += dk
            ref["dv"][b, hk] += dv
    return ref
