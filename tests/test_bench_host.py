"""Host-side accounting of bench.py, checked by brute force on small cases:
the causal pair count P_c behind every TFLOP/s figure (forward 4 d P_c,
backward 10 d P_c), the pairs a block-sparse mask leaves, and the algorithmic
byte counts."""
import numpy as np
import pytest

import bench
import fa2_inputs


def brute_pairs(N, causal, mask=None, block=1):
    q = np.arange(N)[:, None]
    k = np.arange(N)[None, :]
    keep = np.ones((N, N), dtype=bool) if not causal else (k <= q)
    if mask is not None:
        keep &= np.asarray(mask, dtype=bool)[q // block, k // block]
    return int(keep.sum())


@pytest.mark.parametrize("N", [1, 2, 7, 128, 300])
@pytest.mark.parametrize("causal", [True, False])
def test_causal_pairs_and_flops(N, causal):
    w = fa2_inputs.Workload("t", 2, 3, N, 64, "bf16", 0, causal)
    pc = bench.causal_pairs(w)
    assert pc == 2 * 3 * brute_pairs(N, causal)
    f_fwd, f_bwd = bench.flops(w)
    assert f_fwd == 4 * 64 * pc and f_bwd == 10 * 64 * pc


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("causal", [True, False])
def test_block_sparse_pairs(seed, causal):
    block, tiles = 4, 6
    rng = np.random.default_rng(seed)
    mask = (rng.random((tiles, tiles)) < 0.5).astype(np.uint8)
    got = bench.block_sparse_pairs(mask, causal, block)
    assert got == brute_pairs(tiles * block, causal, mask, block)


def test_block_sparse_pairs_all_ones_is_dense():
    ones = np.ones((5, 5), dtype=np.uint8)
    assert bench.block_sparse_pairs(ones, True, 8) == brute_pairs(40, True)
    assert bench.block_sparse_pairs(ones, False, 8) == 40 * 40


def test_alg_bytes_10b_head_shape():
    """Forward: Q, K, V read and O written (bf16) plus L (fp32); backward: Q, K,
    V, O, dO read and dQ, dK, dV written plus L, D and L*log2(e)."""
    w = fa2_inputs.WORKLOADS["10b-b1h36-n4096-d128"]
    t = 36 * 4096 * 128 * 2
    rows = 36 * 4096 * 4
    fwd, bwd = bench.alg_bytes(w)
    assert fwd == 4 * t + rows == 151_584_768
    assert bwd == 8 * t + 3 * rows


@pytest.mark.parametrize("N", [1, 100, 128, 129, 4096])
@pytest.mark.parametrize("causal", [True, False])
def test_single_tile_pairs(N, causal):
    """Causal pairs of the rows whose query tile sees a single key tile (the
    first 128 rows under the causal rule): counted by brute force."""
    w = fa2_inputs.Workload("t", 2, 3, N, 64, "bf16", 0, causal)
    q = np.arange(N)[:, None]
    k = np.arange(N)[None, :]
    brute = int(((k <= q) & (q < 128)).sum()) if causal else 0
    assert bench.single_tile_pairs(w) == 2 * 3 * brute


def test_workload_by_name_covers_fixed_and_sweep_points():
    for w in fa2_inputs.WORKLOADS.values():
        assert fa2_inputs.workload_by_name(w.name) is w
    for w in fa2_inputs.sweep_workloads():
        assert fa2_inputs.workload_by_name(w.name) == w
    for bad in ("sweep-b1h16-n4096-d128-int8", "sweep-b2h16-n4096-d128-fp32", "10b"):
        with pytest.raises(KeyError):
            fa2_inputs.workload_by_name(bad)
