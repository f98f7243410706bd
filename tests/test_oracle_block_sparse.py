"""Pins for the oracle's block-sparse attention ("Notes on flashattention",
section "Block-sparse Flashattention": zero blocks of the block mask are
skipped, i.e. their scores take no part in the softmax; combined with the
causal rule key j is visible to query i iff j <= i and its block is set).

Checked against facts that do not come from these functions: a hand-derived
worked example with every value in closed form (tests/golden/), the dense oracle
(already pinned) for an all-ones mask and, block by block, for a block-diagonal
mask; torch's float64 scaled_dot_product_attention with the element mask the
blocks expand to; central finite differences; and the rule that a query row
seeing no key has O = 0, L = -inf, dQ = 0 and no influence on dK, dV.
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


def element_mask(block_mask, nq, nk, bq, bk, causal):
    m = np.repeat(np.repeat(np.asarray(block_mask, dtype=bool), bq, axis=0), bk, axis=1)[:nq, :nk]
    if causal:
        m &= np.tril(np.ones((nq, nk), dtype=bool))
    return m


def test_worked_example_block_sparse_n4_d2(oracle_mod):
    with open(os.path.join(GOLDEN, "worked_example_block_sparse_n4_d2.json")) as f:
        g = json.load(f)
    inp, exp = g["inputs"], g["expected"]
    q, k, v, do = (np.array(inp[n])[None] for n in ("q", "k", "v", "do"))
    args = (inp["causal"], inp["scale"], np.array(inp["block_mask"]), inp["block_q"], inp["block_k"])
    o, lse = oracle_mod.forward_block_sparse(q, k, v, *args)
    dq, dk, dv = oracle_mod.backward_block_sparse(q, k, v, do, *args)
    tol = g["tolerance"]
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got[0], exp[name], atol=tol, rtol=0, err_msg=name)


@pytest.mark.parametrize("causal", [True, False])
def test_all_ones_mask_is_dense(oracle_mod, causal):
    nq, nk, d, bq, bk = 37, 45, 8, 8, 16
    q, k, v, do = rand((2, nq, d), 1), rand((2, nk, d), 2), rand((2, nk, d), 3), rand((2, nq, d), 4)
    mask = np.ones((math.ceil(nq / bq), math.ceil(nk / bk)), dtype=np.uint8)
    o, lse = oracle_mod.forward_block_sparse(q, k, v, causal, 0.3, mask, bq, bk)
    o_ref, lse_ref = oracle_mod.forward(q, k, v, causal, 0.3)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-13)
    g = oracle_mod.backward_block_sparse(q, k, v, do, causal, 0.3, mask, bq, bk)
    g_ref = oracle_mod.backward(q, k, v, do, causal, 0.3)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_block_diagonal_is_blockwise_dense(oracle_mod):
    """A block-diagonal mask (non-causal) makes each query block attend only to
    its own key block: the dense oracle on each block pair separately."""
    n, d, b = 48, 4, 16
    q, k, v, do = (rand((1, n, d), s) for s in (10, 11, 12, 13))
    mask = np.eye(n // b, dtype=np.uint8)
    o, lse = oracle_mod.forward_block_sparse(q, k, v, False, 0.5, mask, b, b)
    dq, dk, dv = oracle_mod.backward_block_sparse(q, k, v, do, False, 0.5, mask, b, b)
    for t in range(n // b):
        sl = slice(t * b, (t + 1) * b)
        o_r, l_r = oracle_mod.forward(q[:, sl], k[:, sl], v[:, sl], False, 0.5)
        dq_r, dk_r, dv_r = oracle_mod.backward(q[:, sl], k[:, sl], v[:, sl], do[:, sl], False, 0.5)
        np.testing.assert_allclose(o[:, sl], o_r, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[:, sl], l_r, atol=1e-13, rtol=0)
        np.testing.assert_allclose(dq[:, sl], dq_r, atol=1e-12, rtol=0)
        np.testing.assert_allclose(dk[:, sl], dk_r, atol=1e-12, rtol=0)
        np.testing.assert_allclose(dv[:, sl], dv_r, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("seed,bq,bk", [(0, 8, 8), (1, 8, 8), (2, 8, 8), (3, 8, 4), (4, 4, 8)])
def test_against_torch_sdpa_with_element_mask(oracle_mod, causal, seed, bq, bk):
    """Independent library routine: torch SDPA in float64 with autograd, the
    boolean element mask expanded from the blocks (also with different query
    and key block sizes).  Every query block keeps a block on the diagonal
    rows so that every row sees at least one key (SDPA returns NaN for rows
    with none)."""
    nq, nk, d = 40, 40, 8
    rng = np.random.default_rng(300 + seed)
    mask = (rng.random((nq // bq, nk // bk)) < 0.5).astype(np.uint8)
    for a in range(nq // bq):
        mask[a, (a * bq) // bk] = 1              # the block holding key a*bq: row a*bq sees it
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn(1, 1, 40, d, generator=g, dtype=torch.float64) for _ in range(4))
    allowed = torch.from_numpy(element_mask(mask, nq, nk, bq, bk, causal))
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed, scale=0.4)
    ot.backward(do)
    s = (torch.einsum("bhid,bhjd->bhij", q, k) * 0.4).masked_fill(~allowed, float("-inf"))
    o, lse = oracle_mod.forward_block_sparse(q.numpy(), k.numpy(), v.numpy(), causal, 0.4, mask, bq, bk)
    dq, dk, dv = oracle_mod.backward_block_sparse(q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                                  causal, 0.4, mask, bq, bk)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11, rtol=1e-11)


@pytest.mark.parametrize("causal", [True, False])
def test_rows_without_keys(oracle_mod, causal):
    """Query blocks whose mask row is empty: O = 0, L = -inf, dQ = 0, and their
    dO has no effect on dK and dV."""
    nq, nk, d, b = 32, 32, 4, 8
    q, k, v, do = (rand((1, 32, d), s) for s in (20, 21, 22, 23))
    mask = np.tril(np.ones((4, 4), dtype=np.uint8))
    mask[2, :] = 0
    o, lse = oracle_mod.forward_block_sparse(q, k, v, causal, 0.5, mask, b, b)
    assert np.all(o[:, 16:24] == 0) and np.all(np.isneginf(lse[:, 16:24]))
    assert np.all(np.isfinite(lse[:, :16])) and np.all(np.isfinite(lse[:, 24:]))
    dq, dk, dv = oracle_mod.backward_block_sparse(q, k, v, do, causal, 0.5, mask, b, b)
    assert np.all(dq[:, 16:24] == 0)
    do2 = do.copy()
    do2[:, 16:24] = rand((1, 8, d), 99)
    _, dk2, dv2 = oracle_mod.backward_block_sparse(q, k, v, do2, causal, 0.5, mask, b, b)
    np.testing.assert_array_equal(dk, dk2)
    np.testing.assert_array_equal(dv, dv2)


@pytest.mark.parametrize("causal", [True, False])
def test_finite_differences(oracle_mod, causal):
    """Central differences of Phi = sum(dO o O) w.r.t. q, k, v match the
    analytic block-sparse gradients (tiny problem, blocks of 2)."""
    nq, nk, d, b, h = 6, 6, 3, 2, 1e-6
    mask = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], dtype=np.uint8)
    q, k, v, do = rand((1, nq, d), 40), rand((1, nk, d), 41), rand((1, nk, d), 42), rand((1, nq, d), 43)

    def phi(q_, k_, v_):
        o, _ = oracle_mod.forward_block_sparse(q_, k_, v_, causal, 0.7, mask, b, b)
        return float((o * do).sum())

    grads = oracle_mod.backward_block_sparse(q, k, v, do, causal, 0.7, mask, b, b)
    for which, x, g in zip(range(3), (q, k, v), grads):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xs = [q, k, v]
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            xs[which] = xp
            fp = phi(*xs)
            xs[which] = xm
            fm = phi(*xs)
            fd[idx] = (fp - fm) / (2 * h)
        assert np.abs(fd - g).max() <= 1e-7 * max(1.0, np.abs(g).max()), (which, np.abs(fd - g).max())


def test_bad_mask_shape_rejected(oracle_mod):
    q = rand((1, 16, 4), 1)
    with pytest.raises(ValueError):
        oracle_mod.forward_block_sparse(q, q, q, True, 1.0, np.ones((3, 2)), 8, 8)
