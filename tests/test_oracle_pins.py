"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself (a hand-derived worked example, closed forms, invariants, finite
differences, and an independent library routine), chosen so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails at
least one of them.

Sources: CS336 A2 Systems handout section 4.2.2 (Eqs. 4-19, Algorithm 1, the
causal rule of Problem flash_forward (c), the identity D = rowsum(O o dO) =
rowsum(P o dP)); "Notes on flashattention" (Theorem 1's invariants and the
backward derivation of dS through the softmax Jacobian).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- worked example

def test_worked_example_causal_n2_d2(oracle_mod):
    with open(os.path.join(GOLDEN, "worked_example_causal_n2_d2.json")) as f:
        g = json.load(f)
    inp, exp = g["inputs"], g["expected"]
    q, k, v, do = (np.array(inp[n])[None] for n in ("q", "k", "v", "do"))
    o, lse = oracle_mod.forward(q, k, v, inp["causal"], inp["scale"])
    dq, dk, dv = oracle_mod.backward(q, k, v, do, inp["causal"], inp["scale"])
    tol = g["tolerance"]
    np.testing.assert_allclose(o[0], exp["o"], atol=tol, rtol=0)
    np.testing.assert_allclose(lse[0], exp["lse"], atol=tol, rtol=0)
    np.testing.assert_allclose(dq[0], exp["dq"], atol=tol, rtol=0)
    np.testing.assert_allclose(dk[0], exp["dk"], atol=tol, rtol=0)
    np.testing.assert_allclose(dv[0], exp["dv"], atol=tol, rtol=0)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("d", [1, 8, 64])
def test_causal_row0_closed_form(oracle_mod, d):
    """Causal query 0 sees only key 0: O_0 = v_0, L_0 = scale q_0.k_0, dQ_0 = 0."""
    N, scale = 7, 0.37
    q, k, v, do = (rand((2, N, d), s) for s in range(4))
    o, lse = oracle_mod.forward(q, k, v, True, scale)
    dq, dk, dv = oracle_mod.backward(q, k, v, do, True, scale)
    for h in range(2):
        np.testing.assert_allclose(o[h, 0], v[h, 0], atol=1e-14)
        assert abs(lse[h, 0] - scale * float(q[h, 0] @ k[h, 0])) < 1e-13
        np.testing.assert_allclose(dq[h, 0], 0.0, atol=1e-14)
        # The last key is seen only by the last query, with weight P_{N-1,N-1}:
        # dV_{N-1} = P_{N-1,N-1} dO_{N-1}, P_{N-1,N-1} = exp(S_{N-1,N-1} - L_{N-1}).
        p_last = math.exp(scale * float(q[h, -1] @ k[h, -1]) - lse[h, -1])
        np.testing.assert_allclose(dv[h, -1], p_last * do[h, -1], atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_identical_keys_prefix_mean(oracle_mod, causal):
    """All keys equal -> uniform weights over the visible keys:
    O_i = mean of visible v, L_i = scale q_i.k + log(#visible), dQ = 0."""
    N, d, scale = 9, 5, 0.8
    q, v, do = rand((1, N, d), 1), rand((1, N, d), 2), rand((1, N, d), 3)
    kvec = rand((d,), 4)
    k = np.broadcast_to(kvec, (1, N, d)).copy()
    o, lse = oracle_mod.forward(q, k, v, causal, scale)
    dq, _, _ = oracle_mod.backward(q, k, v, do, causal, scale)
    for i in range(N):
        nvis = i + 1 if causal else N
        np.testing.assert_allclose(o[0, i], v[0, :nvis].mean(axis=0), atol=1e-13)
        assert abs(lse[0, i] - (scale * float(q[0, i] @ kvec) + math.log(nvis))) < 1e-12
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)


def test_noncausal_single_key(oracle_mod):
    """N=1: O = v_0, L = scale q.k, dQ = dK = 0, dV = dO."""
    d, scale = 6, 1.3
    q, k, v, do = (rand((3, 1, d), s) for s in range(4))
    o, lse = oracle_mod.forward(q, k, v, False, scale)
    dq, dk, dv = oracle_mod.backward(q, k, v, do, False, scale)
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(lse[:, 0], scale * np.einsum("hd,hd->h", q[:, 0], k[:, 0]),
                               atol=1e-14)
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    np.testing.assert_allclose(dv, do, atol=1e-15)


@pytest.mark.parametrize("causal", [True, False])
def test_identity_values_expose_probabilities(oracle_mod, causal):
    """With V = I (N <= d) the output rows are the attention probabilities:
    rows sum to 1, masked entries are exactly 0, and P_ij / P_i0 =
    exp(scale q_i.(k_j - k_0)) for visible j."""
    N, d, scale = 6, 8, 0.6
    q, k = rand((1, N, d), 10), rand((1, N, d), 11)
    v = np.eye(N, d)[None]
    o, _ = oracle_mod.forward(q, k, v, causal, scale)
    P = o[0, :, :N]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    for i in range(N):
        for j in range(N):
            if causal and j > i:
                assert P[i, j] == 0.0
            else:
                ratio = math.exp(scale * float(q[0, i] @ (k[0, j] - k[0, 0])))
                assert abs(P[i, j] / P[i, 0] - ratio) < 1e-12 * max(1.0, ratio)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [True, False])
def test_shift_invariances(oracle_mod, causal):
    """K -> K + c leaves O unchanged and moves L_i by scale q_i.c;
    V -> V + c moves every O_i by c (the weights sum to one)."""
    N, d, scale = 11, 7, 0.45
    q, k, v = (rand((2, N, d), s) for s in (20, 21, 22))
    c = rand((d,), 23)
    o, lse = oracle_mod.forward(q, k, v, causal, scale)
    o_k, lse_k = oracle_mod.forward(q, k + c, v, causal, scale)
    o_v, lse_v = oracle_mod.forward(q, k, v + c, causal, scale)
    np.testing.assert_allclose(o_k, o, atol=1e-13)
    np.testing.assert_allclose(lse_k, lse + scale * (q @ c), atol=1e-12)
    np.testing.assert_allclose(o_v, o + c, atol=1e-13)
    np.testing.assert_allclose(lse_v, lse, atol=0)


@pytest.mark.parametrize("causal", [True, False])
def test_gradient_invariants(oracle_mod, causal):
    """sum_j dK_j = 0 (shift invariance in K), sum_j dV_j = sum_i dO_i
    (shift in V), and the handout's identity
    D_i = rowsum(O o dO)_i = sum_j P_ij dP_ij."""
    N, d, scale = 13, 6, 0.5
    q, k, v, do = (rand((3, N, d), s) for s in (30, 31, 32, 33))
    o, _ = oracle_mod.forward(q, k, v, causal, scale)
    dq, dk, dv, stats = oracle_mod.backward(q, k, v, do, causal, scale, return_stats=True)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)
    np.testing.assert_allclose(stats[..., 1], (o * do).sum(axis=-1), atol=1e-12)


# ---------------------------------------------------------------- finite differences

def _phi(oracle_mod, q, k, v, do, causal, scale):
    o, _ = oracle_mod.forward(q, k, v, causal, scale)
    return float((o * do).sum())


@pytest.mark.parametrize("N,d", [(1, 1), (2, 4), (3, 16), (5, 4), (8, 16)])
@pytest.mark.parametrize("causal", [True, False])
def test_finite_differences(oracle_mod, N, d, causal):
    """Central differences of Phi = sum(dO o O) w.r.t. every entry of q, k, v
    match the analytic dQ, dK, dV."""
    scale, h = 1.0 / math.sqrt(d), 1e-6
    q, k, v, do = (rand((1, N, d), 100 + s + 10 * N + d) for s in range(4))
    dq, dk, dv = oracle_mod.backward(q, k, v, do, causal, scale)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _phi(oracle_mod, args["q"], args["k"], args["v"], do, causal, scale)
            args[name] = xm
            fm = _phi(oracle_mod, args["q"], args["k"], args["v"], do, causal, scale)
            fd[idx] = (fp - fm) / (2 * h)
        err = np.abs(fd - g).max()
        assert err <= 1e-7 * max(1.0, np.abs(g).max()), (name, err)


# ---------------------------------------------------------------- library cross-check

@pytest.mark.parametrize("B,H,N,d", [(1, 2, 17, 8), (2, 3, 33, 16), (1, 1, 64, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_against_torch_sdpa_float64(oracle_mod, B, H, N, d, causal):
    """Independent library routine: torch's scaled_dot_product_attention in
    float64 on the CPU with autograd; L against torch.logsumexp of the masked
    scores."""
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator().manual_seed(5 + N + d)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4))
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal,
                                                          scale=scale)
    ot.backward(do)
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    lse_t = torch.logsumexp(s, dim=-1)
    o, lse = oracle_mod.forward(q.numpy(), k.numpy(), v.numpy(), causal, scale)
    dq, dk, dv = oracle_mod.backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, scale)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, lse_t.numpy(), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11, rtol=1e-11)


def test_unequal_lengths_against_explicit_mask(oracle_mod):
    """N_q != N_k with the top-left causal rule (key j visible iff j <= i),
    checked against torch's attention with that boolean mask."""
    nq, nk, d, scale = 9, 14, 8, 0.3
    g = torch.Generator().manual_seed(77)
    q = torch.randn(1, 1, nq, d, generator=g, dtype=torch.float64)
    k, v = (torch.randn(1, 1, nk, d, generator=g, dtype=torch.float64) for _ in range(2))
    allowed = torch.ones(nq, nk, dtype=torch.bool).tril()
    ot = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed,
                                                          scale=scale)
    o, _ = oracle_mod.forward(q.numpy(), k.numpy(), v.numpy(), True, scale)
    np.testing.assert_allclose(o, ot.numpy(), atol=1e-12, rtol=1e-12)


# ---------------------------------------------------------------- sampled entry point

@pytest.mark.parametrize("causal", [True, False])
def test_sampled_matches_full(oracle_mod, causal):
    """The per-row sampled entry point returns exactly the full outputs' rows."""
    N, d, scale = 40, 8, 0.35
    q, k, v, do = (rand((1, N, d), s) for s in (50, 51, 52, 53))
    o, lse = oracle_mod.forward(q, k, v, causal, scale)
    dq, dk, dv = oracle_mod.backward(q, k, v, do, causal, scale)
    rows = [0, 3, 17, 39]
    res = oracle_mod.head_sampled(q[0], k[0], v[0], do[0], causal, scale, rows, rows)
    np.testing.assert_array_equal(res["o"], o[0, rows])
    np.testing.assert_array_equal(res["lse"], lse[0, rows])
    np.testing.assert_allclose(res["dq"], dq[0, rows], atol=0, rtol=0)
    np.testing.assert_allclose(res["dk"], dk[0, rows], atol=0, rtol=0)
    np.testing.assert_allclose(res["dv"], dv[0, rows], atol=0, rtol=0)


def test_bad_arguments_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.forward(np.zeros((2, 3)), np.zeros((2, 4)), np.zeros((2, 4)), True, 1.0)
    with pytest.raises(RuntimeError):
        oracle_mod.head_sampled(np.zeros((4, 2)), np.zeros((4, 2)), np.zeros((4, 2)),
                                np.zeros((4, 2)), True, 1.0, [5], [0])
