"""Pins for the grouped-query / multi-query reference used by the GPU parity
tests: H query heads share H_kv key/value heads, query head h reading key/value
head h // (H // H_kv) (the "LLM FLOPs Computation" page, section Extension: GQA:
a group of query heads shares one key and one value head).
The reference runs the oracle per query head and sums dK, dV over a group.

Checked against an independent routine (torch's scaled_dot_product_attention
in float64 on the CPU, K and V broadcast to all query heads by
repeat_interleave, gradients through the broadcast by autograd) and a closed
form (identical query heads within a group multiply dK, dV by the group size).
"""
import math

import numpy as np
import pytest
import torch

from parity_util import grouped_reference


def _rand(B, H, H_kv, N, Nk, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, H_kv, Nk, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, H_kv, Nk, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    return q, k, v, do


@pytest.mark.parametrize("B,H,H_kv,N,Nk,d,causal", [
    (1, 4, 2, 19, 19, 8, True),
    (2, 6, 1, 16, 16, 16, True),     # multi-query
    (1, 4, 4, 12, 12, 8, False),     # one query head per key/value head
    (1, 6, 3, 13, 29, 8, True),      # more keys than queries
    (1, 2, 1, 21, 9, 16, False),     # fewer keys than queries
])
def test_grouped_reference_against_sdpa_broadcast(oracle_mod, B, H, H_kv, N, Nk, d, causal):
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = _rand(B, H, H_kv, N, Nk, d, seed=7 + H + N + Nk)
    ref = grouped_reference(oracle_mod, q, k, v, do, causal, scale)
    grp = H // H_kv
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    kb, vb = kt.repeat_interleave(grp, dim=1), vt.repeat_interleave(grp, dim=1)
    mask = None
    if causal:  # key j visible to query i iff j <= i (top-left aligned)
        mask = torch.ones(N, Nk, dtype=torch.bool).tril()
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kb, vb, attn_mask=mask, scale=scale)
    ot.backward(do)
    np.testing.assert_allclose(ref["o"], ot.detach().numpy(), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(ref["dq"], qt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(ref["dk"], kt.grad.numpy(), atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(ref["dv"], vt.grad.numpy(), atol=1e-11, rtol=1e-11)
    s = torch.einsum("bhid,bhjd->bhij", q, k.repeat_interleave(grp, dim=1)) * scale
    if causal:
        s = s.masked_fill(~mask, float("-inf"))
    np.testing.assert_allclose(ref["lse"], torch.logsumexp(s, dim=-1).numpy(), atol=1e-12, rtol=1e-12)


def test_identical_heads_scale_key_value_gradients(oracle_mod):
    """All query heads of a group equal (same q, same dO): each contributes the
    same dK, dV, so the shared head's gradients are the group size times those
    of one head, and every head's O, L, dQ are equal."""
    B, H, H_kv, N, d = 1, 6, 2, 17, 8
    scale = 0.3
    q1, k, v, do1 = _rand(B, 1, H_kv, N, N, d, seed=3)
    q, do = q1.expand(B, H, N, d).contiguous(), do1.expand(B, H, N, d).contiguous()
    ref = grouped_reference(oracle_mod, q, k, v, do, True, scale)
    for hk in range(H_kv):
        single = grouped_reference(oracle_mod, q1, k[:, hk:hk + 1], v[:, hk:hk + 1], do1, True, scale)
        np.testing.assert_allclose(ref["dk"][:, hk], 3 * single["dk"][:, 0], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(ref["dv"][:, hk], 3 * single["dv"][:, 0], rtol=1e-13, atol=1e-13)
        for h in range(3 * hk, 3 * hk + 3):
            np.testing.assert_array_equal(ref["o"][:, h], single["o"][:, 0])
            np.testing.assert_array_equal(ref["dq"][:, h], single["dq"][:, 0])


def test_wrong_head_map_is_caught(oracle_mod):
    """A plausible mistake in the head map (h % H_kv instead of h // group)
    changes the results, so the SDPA comparison above would reject it."""
    B, H, H_kv, N, d = 1, 4, 2, 11, 8
    q, k, v, do = _rand(B, H, H_kv, N, N, d, seed=11)
    ref = grouped_reference(oracle_mod, q, k, v, do, True, 0.5)
    perm = torch.tensor([0, 2, 1, 3])   # reorders heads so h // 2 reads what h % 2 would
    alt = grouped_reference(oracle_mod, q[:, perm], k, v, do[:, perm], True, 0.5)
    assert not np.allclose(ref["dk"], alt["dk"])
