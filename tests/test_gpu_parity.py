"""Parity of the CUDA path (called through the C ABI via the binding) with the
fp64 oracle on identical seeded inputs.

Small shapes are compared in full (all of O, L, dQ, dK, dV), spanning several
128-row tiles, ragged tails, N < one tile, every supported head dim, causal
and full attention.  The named workloads (the model-table head shapes) run at
full size in the launch configuration the benchmark uses; their first and
last heads are compared in full.

Tolerance per element: |gpu - ref| <= atol + rtol |ref| with atol = rtol =
1e-2 for bf16 inputs and 2e-3 for fp32 (TF32 tensor-core) inputs.
"""
import numpy as np
import pytest
import torch

import fa2_inputs
from parity_util import assert_close, default_scale, gpu_fwd_bwd, to64

pytestmark = pytest.mark.gpu

SMALL = [
    # (B, H, N, d)
    (1, 2, 128, 64),
    (2, 2, 256, 64),
    (1, 2, 384, 128),
    (1, 2, 200, 64),     # ragged tail
    (1, 1, 1, 64),       # one row
    (1, 2, 64, 32),      # shorter than one tile
    (1, 2, 300, 128),
    (1, 2, 256, 80),
    (1, 2, 320, 16),
    (2, 1, 513, 32),
]


def _oracle(oracle_mod, inp, causal, scale, backward=True):
    q, k, v = (to64(inp[n].float()) for n in ("q", "k", "v"))
    o, lse = oracle_mod.forward(q, k, v, causal, scale)
    res = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = oracle_mod.backward(q, k, v, to64(inp["do"].float()), causal, scale)
        res.update(dq=dq, dk=dk, dv=dv)
    return res


@pytest.mark.parametrize("mode", ["two-pass", "one-pass"])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("B,H,N,d", SMALL)
def test_bf16_small_full_parity(oracle_mod, B, H, N, d, causal, mode):
    """bf16 inputs, every output in full; the backward in its two-pass form
    (FA2_BWD_DETERMINISTIC) and its one-pass form (FA2_BWD_ONE_PASS: one pass
    over key tiles wherever there is more than one key tile)."""
    inp = fa2_inputs.make_inputs(B, H, N, d, "bf16", seed=11 + N + d)
    scale = default_scale(d)
    got = gpu_fwd_bwd(inp, causal, scale, mode=mode)
    ref = _oracle(oracle_mod, inp, causal, scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert_close(to64(got[name]), ref[name], "bf16", name)


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("B,H,N,d", SMALL)
def test_fp32_small_full_parity(oracle_mod, B, H, N, d, causal):
    """fp32 inputs (TF32 tensor-core MMAs): forward and backward in full."""
    inp = fa2_inputs.make_inputs(B, H, N, d, "fp32", seed=17 + N + d)
    scale = default_scale(d)
    got = gpu_fwd_bwd(inp, causal, scale)
    ref = _oracle(oracle_mod, inp, causal, scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert_close(to64(got[name]), ref[name], "fp32", name)


@pytest.mark.parametrize("mode", ["two-pass", "one-pass"])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("B,H,N,d", SMALL)
def test_fp16_small_full_parity(oracle_mod, B, H, N, d, causal, mode):
    """fp16 inputs (kind::f16 MMAs with fp16 operands): forward and backward in full."""
    inp = fa2_inputs.make_inputs(B, H, N, d, "fp16", seed=23 + N + d)
    scale = default_scale(d)
    got = gpu_fwd_bwd(inp, causal, scale, mode=mode)
    ref = _oracle(oracle_mod, inp, causal, scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert_close(to64(got[name]), ref[name], "fp16", name)


def test_fp16_10b_shape_heads(oracle_mod):
    """The 10B head shape (B=1, H=36, N=4096, d=128) with fp16 inputs; first and
    last head compared in full."""
    w = fa2_inputs.WORKLOADS["10b-b1h36-n4096-d128"]
    inp = fa2_inputs.make_inputs(w.B, w.H, w.N, w.d, "fp16", seed=w.seed)
    got = gpu_fwd_bwd(inp, w.causal, w.scale)
    for hh in (0, w.H - 1):
        q, k, v, do = (to64(inp[n][0, hh].float()) for n in ("q", "k", "v", "do"))
        o, lse = oracle_mod.forward(q, k, v, w.causal, w.scale)
        dq, dk, dv = oracle_mod.backward(q, k, v, do, w.causal, w.scale)
        for name, ref in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            e = assert_close(to64(got[name][0, hh]), ref, "fp16", f"{name}[head {hh}]")
            print(f"ERR fp16-10b head {hh} {name} max_abs {e:.3e}")


@pytest.mark.parametrize("scale", [0.09, 0.14, 0.2])
def test_nondefault_scale(oracle_mod, scale):
    """A scale other than 1/sqrt(d) must enter S, dQ and dK.  At d = 64 the
    default is 0.125; 0.2 is 1.6 times sharper, and over six seeds at N = 256
    and 640 its worst dQ / dK element used 0.84 of the bound."""
    inp = fa2_inputs.make_inputs(1, 2, 256, 64, "bf16", seed=5)
    got = gpu_fwd_bwd(inp, True, scale)
    ref = _oracle(oracle_mod, inp, True, scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert_close(to64(got[name]), ref[name], "bf16", name)


@pytest.mark.xfail(strict=True, raises=AssertionError,
                   reason="16-bit backward roundings (D from the 16-bit O, 16-bit dS) "
                          "pass the bound at 3.2x the default scale")
def test_sharp_scale_known_exceedance(oracle_mod):
    """The known limit of the 16-bit backward, pinned: at scale 0.4 (3.2 times
    the default 1/sqrt(64)) the softmax is sharp enough that the backward's
    roundings (D = rowsum(O o dO) taken from the 16-bit O, dS rounded to 16 bits
    before the dQ MMA) move a few dQ elements past the 1e-2 bound (this seed:
    3.9 times the bound at row 155 of head 1; O and L stay inside it, checked by
    the test below).  A change that removes the exceedance turns this into an unexpected
    pass, which fails the run until the pin is updated."""
    inp = fa2_inputs.make_inputs(1, 2, 256, 64, "bf16", seed=3)
    got = gpu_fwd_bwd(inp, True, 0.4, mode="two-pass")
    ref = _oracle(oracle_mod, inp, True, 0.4)
    assert_close(to64(got["dq"]), ref["dq"], "bf16", "dq")


def test_sharp_scale_forward(oracle_mod):
    """The forward at the same sharp scale (0.4, d = 64) stays inside the bound:
    the exceedance above belongs to the backward."""
    inp = fa2_inputs.make_inputs(1, 2, 256, 64, "bf16", seed=3)
    got = gpu_fwd_bwd(inp, True, 0.4, do_backward=False)
    ref = _oracle(oracle_mod, inp, True, 0.4, backward=False)
    for name in ("o", "lse"):
        assert_close(to64(got[name]), ref[name], "bf16", name)


BF16_WORKLOADS = [w for w in fa2_inputs.WORKLOADS.values() if w.dtype == "bf16"]


@pytest.mark.parametrize("mode", ["two-pass", "one-pass"])
@pytest.mark.parametrize("w", BF16_WORKLOADS, ids=[w.name for w in BF16_WORKLOADS])
def test_workload_full_heads_parity(oracle_mod, w, mode):
    """Full-size workload on the GPU (the benchmark's launch configuration in
    the default mode); the first and the last head are compared element by
    element (all rows of O, L, dQ, dK, dV) with the oracle."""
    inp = fa2_inputs.workload_inputs(w)
    got = gpu_fwd_bwd(inp, w.causal, w.scale, mode=mode)
    heads = sorted({0, w.heads - 1})
    for hh in heads:
        b, h = divmod(hh, w.H)
        q, k, v, do = (to64(inp[n][b, h].float()) for n in ("q", "k", "v", "do"))
        o, lse = oracle_mod.forward(q, k, v, w.causal, w.scale)
        dq, dk, dv = oracle_mod.backward(q, k, v, do, w.causal, w.scale)
        for name, ref in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            e = assert_close(to64(got[name][b, h]), ref, w.dtype, f"{name}[head {hh}]")
            print(f"ERR {w.name} {mode} head {hh} {name} max_abs {e:.3e}")


def test_fp32_workload_full(oracle_mod):
    """The fp32 model-table workload (B=2, H=4, N=128, d=64), every output in full."""
    w = fa2_inputs.WORKLOADS["fp32-b2h4-n128-d64"]
    inp = fa2_inputs.workload_inputs(w)
    got = gpu_fwd_bwd(inp, w.causal, w.scale)
    ref = _oracle(oracle_mod, inp, w.causal, w.scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        e = assert_close(to64(got[name]), ref[name], "fp32", name)
        print(f"ERR {w.name} all heads {name} max_abs {e:.3e}")


def test_outputs_stay_in_bounds():
    """Outputs written into the middle of NaN-filled buffers: the guard
    regions before and after each output must be untouched."""
    import causal_attention_fa2_b200 as fa2
    B, H, N, d = 1, 3, 200, 80
    dev = torch.device("cuda", 0)
    inp = fa2_inputs.make_inputs(B, H, N, d, "bf16", seed=3)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    pad = 256
    numel = B * H * N * d

    def guarded(n, dtype):
        buf = torch.full((n + 2 * pad,), float("nan"), dtype=dtype, device=dev)
        return buf, buf[pad:pad + n]

    ob, o = guarded(numel, torch.bfloat16)
    lb, lse = guarded(B * H * N, torch.float32)
    o = o.view(B, H, N, d)
    lse = lse.view(B, H, N)
    fa2.forward(q, k, v, causal=True, out=o, lse=lse)
    grads = [guarded(numel, torch.bfloat16) for _ in range(3)]
    dq, dk, dv = (g[1].view(B, H, N, d) for g in grads)
    fa2.backward(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for buf in [ob, lb] + [g[0] for g in grads]:
        assert torch.isnan(buf[:pad].float()).all() and torch.isnan(buf[-pad:].float()).all()
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t.float()).all()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_forward_and_backward_deterministic(dtype):
    """The forward, and the backward in its two-pass form, give the same bits on
    every run; in the one-pass form dK and dV do too, while dQ (summed by fp32
    reduce-add across key tiles) stays within a few units in the last place of
    its 16-bit rounding."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    inp = fa2_inputs.make_inputs(2, 4, 640, 128, dtype, seed=9)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o1, l1 = fa2.forward(q, k, v)
    o2, l2 = fa2.forward(q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = fa2.backward(q, k, v, o1, l1, do, mode="two-pass")
    g2 = fa2.backward(q, k, v, o1, l1, do, mode="two-pass")
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))
    h1 = fa2.backward(q, k, v, o1, l1, do, mode="one-pass")
    h2 = fa2.backward(q, k, v, o1, l1, do, mode="one-pass")
    torch.cuda.synchronize()
    assert torch.equal(h1[1], h2[1]) and torch.equal(h1[2], h2[2])
    torch.testing.assert_close(h1[0].float(), h2[0].float(), atol=1e-3, rtol=1e-2)
    torch.testing.assert_close(h1[0].float(), g1[0].float(), atol=1e-3, rtol=1e-2)


@pytest.mark.parametrize("B,H,N,d,dtype", [(1, 8, 2048, 128, "bf16"), (2, 4, 1024, 64, "bf16"),
                                              (1, 4, 1024, 16, "fp32"), (1, 4, 1024, 32, "fp32"),
                                              (1, 4, 1024, 64, "fp32"), (1, 4, 1024, 128, "fp32")])
def test_two_pass_backward_repeats_bitwise(B, H, N, d, dtype):
    """Twelve back-to-back runs of the two-pass backward give the same bits:
    a check for races between the kernels' warp roles (ping-pong groups, double
    buffers, parted stages), which would show as run-to-run differences."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    inp = fa2_inputs.make_inputs(B, H, N, d, dtype, seed=77 + d)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v)
    ref = fa2.backward(q, k, v, o, lse, do, mode="two-pass")
    runs = [fa2.backward(q, k, v, o, lse, do, mode="two-pass") for _ in range(11)]
    torch.cuda.synchronize()
    for g in runs:
        assert all(torch.equal(a, b) for a, b in zip(ref, g))


def test_autograd_function_matches_direct_calls():
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    inp = fa2_inputs.make_inputs(1, 2, 256, 64, "bf16", seed=21)
    q, k, v = (inp[n].to(dev).requires_grad_(True) for n in ("q", "k", "v"))
    do = inp["do"].to(dev)
    o = fa2.flash_attention(q, k, v, is_causal=True)
    o.backward(do)
    o_ref, lse = fa2.forward(q.detach(), k.detach(), v.detach(), causal=True)
    dq, dk, dv = fa2.backward(q.detach(), k.detach(), v.detach(), o_ref, lse, do, causal=True)
    assert torch.equal(o.detach(), o_ref)
    # dQ of the one-pass backward is summed by reduce-add: same value, bits may differ.
    assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)
    torch.testing.assert_close(q.grad.float(), dq.float(), atol=1e-3, rtol=1e-2)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("is_causal", [None, True], ids=["default", "causal"])
def test_autograd_function_against_oracle(oracle_mod, is_causal, dtype):
    """FlashAttention2Function.apply (the handout's interface) against the
    oracle: O from forward(ctx, Q, K, V, is_causal) and dQ, dK, dV from
    backward(ctx, dO) through torch.autograd.  ``None`` leaves is_causal at the
    interface's default, False (full attention)."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    B, H, N, d = 1, 3, 300, 64
    inp = fa2_inputs.make_inputs(B, H, N, d, dtype, seed=41 + (0 if is_causal is None else 1))
    q, k, v = (inp[n].to(dev).requires_grad_(True) for n in ("q", "k", "v"))
    do = inp["do"].to(dev)
    if is_causal is None:
        o = fa2.FlashAttention2Function.apply(q, k, v)
    else:
        o = fa2.FlashAttention2Function.apply(q, k, v, is_causal)
    o.backward(do)
    torch.cuda.synchronize()
    ref = _oracle(oracle_mod, inp, bool(is_causal), default_scale(d))
    for name, got in (("o", o), ("dq", q.grad), ("dk", k.grad), ("dv", v.grad)):
        assert_close(to64(got), ref[name], dtype, f"autograd {name}")


def test_device_status_clean():
    import causal_attention_fa2_b200 as fa2
    torch.cuda.synchronize()
    assert fa2.last_device_status() == 0
