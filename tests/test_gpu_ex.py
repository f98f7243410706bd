"""fa2_forward_ex / fa2_backward_ex: grouped-query and multi-query attention
(H query heads sharing H_kv key/value heads; query head h uses key/value head
h // (H // H_kv)) and query / key lengths N != Nk (causal: key j visible to
query i iff j <= i).

Reference: the oracle run per query head with that head's shared K and V
(the oracle takes separate query and key lengths); dK and dV of a key/value
head are the sums of the per-query-head oracle gradients over the query
heads sharing it (the chain rule through the broadcast of K and V)."""
import ctypes

import numpy as np
import pytest
import torch

import fa2_inputs
from parity_util import assert_close, default_scale, grouped_reference, to64

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, H_kv, N, Nk, d, dtype, causal)
    (1, 4, 2, 300, 300, 64, "bf16", True),
    (2, 6, 1, 256, 256, 128, "bf16", True),      # multi-query
    (1, 8, 4, 1000, 1000, 80, "bf16", True),
    (1, 4, 2, 384, 384, 128, "bf16", False),
    (1, 4, 1, 200, 200, 32, "fp16", True),
    (1, 4, 2, 200, 200, 64, "fp32", True),
    (1, 6, 3, 160, 160, 16, "fp32", False),
    # different query and key lengths
    (1, 2, 2, 200, 333, 64, "bf16", True),       # keys past the last query: zero dK, dV
    (1, 2, 2, 300, 129, 128, "bf16", True),
    (2, 2, 2, 128, 1000, 64, "bf16", False),
    (1, 4, 2, 513, 64, 80, "bf16", True),
    (1, 2, 1, 170, 390, 32, "fp16", True),
    (1, 2, 2, 150, 400, 64, "fp32", True),
    (1, 2, 2, 260, 100, 128, "fp32", False),
    # fp32 at d = 128 (operands in tensor memory) with grouped heads and ragged lengths
    (1, 4, 2, 300, 257, 128, "fp32", True),
    (1, 3, 1, 129, 300, 128, "fp32", False),
]


def _inputs(B, H, H_kv, N, Nk, d, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    dt = fa2_inputs.DTYPES[dtype]
    q = torch.randn((B, H, N, d), generator=g).to(dt)
    k = torch.randn((B, H_kv, Nk, d), generator=g).to(dt)
    v = torch.randn((B, H_kv, Nk, d), generator=g).to(dt)
    do = torch.randn((B, H, N, d), generator=g).to(dt)
    return q, k, v, do


@pytest.mark.parametrize("B,H,H_kv,N,Nk,d,dtype,causal", CASES)
def test_ex_parity(oracle_mod, B, H, H_kv, N, Nk, d, dtype, causal):
    q, k, v, do = _inputs(B, H, H_kv, N, Nk, d, dtype, seed=131 + N + d + H_kv + Nk)
    _check_against_oracle(oracle_mod, q, k, v, do, causal, dtype, f"ex B={B} H={H} H_kv={H_kv} N={N} Nk={Nk} d={d} {dtype}")


def test_mqa_early_row_regression(oracle_mod):
    """The input on which dQ of causal query row 1 once exceeded the bound
    (0.0169 against 0.0107): multi-query bf16, B=2, H=6, H_kv=1, N=256, d=128,
    inputs drawn with seed 31 + N + d + H_kv = 416.  Row 1 sees two keys, so
    dS_1j is of the order of |dP|; the kernels now take D of the first query
    tile from P and dP and pass its dS in two 16-bit parts.  Same bound as every
    other case."""
    B, H, H_kv, N, d = 2, 6, 1, 256, 128
    q, k, v, do = _inputs(B, H, H_kv, N, N, d, "bf16", seed=31 + N + d + H_kv)
    _check_against_oracle(oracle_mod, q, k, v, do, True, "bf16", "mqa-regression seed 416")


def _check_against_oracle(oracle_mod, q, k, v, do, causal, dtype, label):
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    B, H, N, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    scale = default_scale(d)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa2.forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa2.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert dk.shape == k.shape and dv.shape == v.shape
    ref = grouped_reference(oracle_mod, q, k, v, do, causal, scale)
    if causal and Nk > N:
        # No query reaches keys N .. Nk-1: their gradients are exactly zero.
        assert not dk[:, :, N:].any() and not dv[:, :, N:].any()
    # dK and dV of a key/value head sum the gradients of the `group` query heads
    # that share it.  Each head's part carries its own, independent rounding (P
    # and dS are rounded to the input type per head), so the absolute error of
    # the sum grows like sqrt(group): the bound is sqrt(group) * atol + rtol |ref|
    # (the per-element bound itself for multi-head attention).
    grp = H // H_kv
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        err = np.abs(to64(got) - ref[name])
        tol = TOLS[dtype]
        widen = np.sqrt(grp) if name in ("dk", "dv") else 1.0
        bound = widen * tol + tol * np.abs(ref[name])
        print(f"RATIO {label} {name} {float((err / (tol + tol * np.abs(ref[name]))).max()):.3f} "
              f"(of the widened bound {float((err / bound).max()):.3f})")
        assert np.isfinite(to64(got)).all(), name
        assert (err <= bound).all(), (name, float(err.max()), float((err / bound).max()))
    assert fa2.last_device_status() == 0


TOLS = {"bf16": 1e-2, "fp16": 1e-2, "fp32": 2e-3}


def test_ex_with_mha_shapes_is_bitwise_mha():
    """fa2_forward_ex / fa2_backward_ex with H_kv = H and Nk = N give the bits
    of fa2_forward / fa2_backward."""
    import causal_attention_fa2_b200 as fa2
    from causal_attention_fa2_b200 import _native
    lib = _native.lib()
    dev = torch.device("cuda", 0)
    B, H, N, d = 1, 4, 333, 64
    inp = fa2_inputs.make_inputs(B, H, N, d, "bf16", seed=77)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = default_scale(d)
    o, lse = fa2.forward(q, k, v, causal=True, scale=scale)
    ref = fa2.backward(q, k, v, o, lse, do, causal=True, scale=scale)
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fa2_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), lse2.data_ptr(),
                              B, H, H, N, N, d, 1, scale, 0, s) == 0
    ws = torch.empty(fa2.backward_workspace_bytes(B, H, N, d, q.dtype), dtype=torch.uint8, device=dev)
    g = [torch.empty_like(q) for _ in range(3)]
    assert lib.fa2_backward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               do.data_ptr(), g[0].data_ptr(), g[1].data_ptr(), g[2].data_ptr(),
                               B, H, H, N, N, d, 1, scale, 0, ws.data_ptr(), ws.numel(), s) == 0
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    # dK, dV bitwise; dQ of the one-pass form is summed by reduce-add (order-dependent bits).
    assert torch.equal(ref[1], g[1]) and torch.equal(ref[2], g[2])
    torch.testing.assert_close(ref[0].float(), g[0].float(), atol=1e-3, rtol=1e-2)


def test_gqa_backward_deterministic():
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in _inputs(2, 8, 2, 512, 700, 128, "bf16", seed=5))
    o, lse = fa2.forward(q, k, v)
    g1 = fa2.backward(q, k, v, o, lse, do, mode="two-pass")
    g2 = fa2.backward(q, k, v, o, lse, do, mode="two-pass")
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))
