"""Block-sparse attention (fa2_forward_block_sparse / fa2_backward_block_sparse):
blocks of 128 query rows x 128 key rows whose mask byte is zero are skipped;
with causal, key j is visible to query i iff j <= i and its block is set.  Rows
that see no key: O = 0, L = -inf, dQ = 0, no contribution to dK, dV.

Reference: the oracle's block-sparse functions run per query head with that
head's key/value head; dK, dV of a key/value head sum over the query heads
sharing it.  Masks are seeded inputs (random density 1/2 with some empty block
rows, diagonal, band, a pattern where the two query tiles of one forward CTA
differ, and the empty mask)."""
import numpy as np
import pytest
import torch

import fa2_inputs
from parity_util import TOL, default_scale, to64

pytestmark = pytest.mark.gpu

BLOCK = 128


def _mask(kind, nq_t, nk_t, seed):
    rng = np.random.default_rng(seed)
    if kind == "random":
        m = (rng.random((nq_t, nk_t)) < 0.5).astype(np.uint8)
        m[rng.integers(0, nq_t)] = 0                       # one empty block row
        return m
    if kind == "diag":
        return np.eye(nq_t, nk_t, dtype=np.uint8)
    if kind == "band":                                     # each query tile sees itself and the tile before
        return (np.eye(nq_t, nk_t, dtype=np.uint8) + np.eye(nq_t, nk_t, k=-1, dtype=np.uint8)).clip(0, 1)
    if kind == "pair_split":                               # tiles 2t and 2t+1 differ
        m = np.zeros((nq_t, nk_t), dtype=np.uint8)
        for i in range(nq_t):
            if i % 2 == 0:
                m[i, 0] = 1
            else:
                m[i, min(i, nk_t - 1)] = 1
                m[i, max(0, i - 2)] = 1
        return m
    if kind == "empty":
        return np.zeros((nq_t, nk_t), dtype=np.uint8)
    if kind == "ones":
        return np.ones((nq_t, nk_t), dtype=np.uint8)
    if kind == "mostly_ones":                              # long rows / columns with a few holes
        m = np.ones((nq_t, nk_t), dtype=np.uint8)
        if nk_t > 8:
            for i in range(nq_t):
                m[i, rng.choice(nk_t, 3, replace=False)] = 0
        if nq_t > 8:
            for j in range(nk_t):
                m[rng.choice(nq_t, 3, replace=False), j] = 0
        return m
    raise ValueError(kind)


def _inputs(B, H, H_kv, N, Nk, d, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    dt = fa2_inputs.DTYPES[dtype]
    q = torch.randn((B, H, N, d), generator=g).to(dt)
    k = torch.randn((B, H_kv, Nk, d), generator=g).to(dt)
    v = torch.randn((B, H_kv, Nk, d), generator=g).to(dt)
    do = torch.randn((B, H, N, d), generator=g).to(dt)
    return q, k, v, do


CASES = [
    # (B, H, H_kv, N, Nk, d, dtype, causal, mask kind)
    (1, 2, 2, 640, 640, 64, "bf16", True, "random"),
    (1, 2, 2, 640, 640, 128, "bf16", False, "random"),
    (1, 4, 2, 600, 700, 80, "fp16", True, "random"),
    (1, 2, 2, 700, 450, 32, "bf16", False, "random"),
    (2, 2, 1, 512, 512, 128, "bf16", True, "diag"),
    (1, 2, 2, 1024, 1024, 128, "bf16", True, "band"),
    (1, 2, 2, 768, 768, 64, "bf16", True, "pair_split"),
    (1, 2, 2, 768, 640, 16, "fp16", False, "pair_split"),
    (1, 2, 2, 384, 384, 32, "bf16", True, "empty"),
    # More than 512 tiles on one side (520 x 128 rows), about 517 set blocks per
    # row (forward, dQ pass) or per column (dK/dV pass): past the shared-memory
    # tile list, the kernels walk the mask.
    (1, 2, 2, 128, 520 * 128, 16, "bf16", False, "mostly_ones"),
    (1, 2, 2, 520 * 128, 1024, 16, "bf16", False, "mostly_ones"),
    (1, 2, 1, 200, 520 * 128 - 37, 32, "fp16", False, "mostly_ones"),
    # fp32 inputs (TF32 kernels, streamed in sub-tiles of W rows: every set block
    # is visited as its 128 / W sub-tiles).
    (1, 2, 2, 640, 640, 64, "fp32", True, "random"),
    (1, 4, 2, 600, 700, 128, "fp32", False, "random"),
    (1, 2, 2, 768, 768, 32, "fp32", True, "pair_split"),
    (1, 2, 2, 700, 450, 16, "fp32", False, "band"),
    (1, 2, 2, 384, 384, 80, "fp32", True, "empty"),
]


@pytest.mark.parametrize("B,H,H_kv,N,Nk,d,dtype,causal,kind", CASES)
def test_block_sparse_parity(oracle_mod, B, H, H_kv, N, Nk, d, dtype, causal, kind):
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    nq_t, nk_t = -(-N // BLOCK), -(-Nk // BLOCK)
    mask = _mask(kind, nq_t, nk_t, seed=N + Nk + d)
    q, k, v, do = _inputs(B, H, H_kv, N, Nk, d, dtype, seed=500 + N + Nk + d)
    if N > 512 * BLOCK:
        # Every dK, dV element here sums about 66 000 query rows, and its error
        # follows the largest values (about 0.3 % of max |dK|, |dV| in the dense
        # kernels as well, whose bits the mask walk reproduces for a mask of ones):
        # with unit-variance dO those reach 15-20 and the error the absolute part
        # of the bound.  dK and dV are linear in dO, so dO / 8 keeps the check
        # element-wise at the same bound.
        do = (do.float() / 8).to(do.dtype)
    scale = default_scale(d)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    md = torch.from_numpy(mask).to(dev)
    o, lse = fa2.forward(qd, kd, vd, causal=causal, scale=scale, block_mask=md)
    dq, dk, dv = fa2.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale, block_mask=md)
    torch.cuda.synchronize()
    assert fa2.last_device_status() == 0

    grp = H // H_kv
    ref = {"o": np.zeros((B, H, N, d)), "lse": np.zeros((B, H, N)), "dq": np.zeros((B, H, N, d)),
           "dk": np.zeros((B, H_kv, Nk, d)), "dv": np.zeros((B, H_kv, Nk, d))}
    for b in range(B):
        for h in range(H):
            hk = h // grp
            qh, kh, vh, doh = (to64(t.float()) for t in (q[b, h], k[b, hk], v[b, hk], do[b, h]))
            ro, rl = oracle_mod.forward_block_sparse(qh, kh, vh, causal, scale, mask, BLOCK, BLOCK)
            rdq, rdk, rdv = oracle_mod.backward_block_sparse(qh, kh, vh, doh, causal, scale, mask,
                                                             BLOCK, BLOCK)
            ref["o"][b, h], ref["lse"][b, h], ref["dq"][b, h] = ro, rl, rdq
            ref["dk"][b, hk] += rdk
            ref["dv"][b, hk] += rdv

    atol, rtol = TOL[dtype]
    empty = np.isneginf(ref["lse"])                       # rows that see no key
    got = {n: to64(t) for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    assert np.array_equal(np.isneginf(got["lse"]), empty), "rows with L = -inf differ"
    assert np.all(got["o"][empty] == 0) and np.all(got["dq"][empty] == 0)
    for name in ("o", "lse", "dq", "dk", "dv"):
        g, r = got[name], ref[name]
        if name in ("o", "lse", "dq"):
            keep = ~empty
            g, r = g[keep], r[keep]
        assert np.isfinite(g).all(), f"{name}: non-finite values"
        # dK, dV sum `grp` query heads' independently rounded parts: atol * sqrt(grp)
        scale_t = np.sqrt(grp) if name in ("dk", "dv") else 1
        err = np.abs(g - r)
        bound = scale_t * atol + rtol * np.abs(r)
        assert (err <= bound).all(), (name, float(err.max()), int((err > bound).sum()))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_all_ones_mask_is_bitwise_dense(dtype):
    """A mask of ones gives the bits of the dense entry points (block masks
    take the two-pass backward, so the dense one runs with FA2_BWD_DETERMINISTIC)."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    B, H, N, d = 1, 4, 700, 64
    q, k, v, do = (t.to(dev) for t in _inputs(B, H, H, N, N, d, dtype, seed=9))
    ones = torch.ones(-(-N // BLOCK), -(-N // BLOCK), dtype=torch.bool, device=dev)
    for causal in (True, False):
        o, lse = fa2.forward(q, k, v, causal=causal)
        o2, lse2 = fa2.forward(q, k, v, causal=causal, block_mask=ones)
        g = fa2.backward(q, k, v, o, lse, do, causal=causal, mode="two-pass")
        g2 = fa2.backward(q, k, v, o, lse, do, causal=causal, block_mask=ones)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
        assert all(torch.equal(a, b) for a, b in zip(g, g2))


@pytest.mark.parametrize("B,H,H_kv,N,Nk,d,causal", [
    (1, 1, 1, 520 * 128, 520 * 128, 16, True),     # query-tile pairs, up to 520 steps per row / column
    (1, 148, 1, 256, 520 * 128, 16, False),        # 148 query-tile pairs of 520 key tiles each
])
def test_all_ones_mask_past_the_tile_list_is_bitwise_dense(B, H, H_kv, N, Nk, d, causal):
    """More than 512 tiles per side: the kernels walk a mask of ones and must
    give the dense entry points' bits."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(N + Nk + H)
    q, do = (torch.randn((B, H, N, d), generator=g, device=dev).to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn((B, H_kv, Nk, d), generator=g, device=dev).to(torch.bfloat16) for _ in range(2))
    ones = torch.ones(-(-N // BLOCK), -(-Nk // BLOCK), dtype=torch.bool, device=dev)
    o, lse = fa2.forward(q, k, v, causal=causal)
    o2, lse2 = fa2.forward(q, k, v, causal=causal, block_mask=ones)
    grads = fa2.backward(q, k, v, o, lse, do, causal=causal, mode="two-pass")
    grads2 = fa2.backward(q, k, v, o, lse, do, causal=causal, block_mask=ones)
    torch.cuda.synchronize()
    assert fa2.last_device_status() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    for a, b in zip(grads, grads2):
        assert torch.equal(a, b)


def test_block_sparse_deterministic():
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in _inputs(1, 4, 2, 1024, 1024, 128, "bf16", seed=3))
    m = torch.from_numpy(_mask("random", 8, 8, seed=4)).to(dev)
    o, lse = fa2.forward(q, k, v, block_mask=m)
    g1 = fa2.backward(q, k, v, o, lse, do, block_mask=m)
    g2 = fa2.backward(q, k, v, o, lse, do, block_mask=m)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))
