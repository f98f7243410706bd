"""Parity on points of the causal sequence-length x head-dimension sweep
(B=1, H=16, N = 128 ... 32768, d in {16, 32, 64, 128}, bf16 and fp32 inputs),
in the launch configuration the benchmark uses.

Points with N <= 1024 are compared in full.  Longer points are run in full on
the GPU and checked on two heads (the first and the last; one head at
N = 32768): O, L and dQ on seeded query rows, dK and dV on seeded key rows,
always including the first and the last row, against the oracle's per-row
evaluation of the same head."""
import pytest

import fa2_inputs
from parity_util import assert_close, gpu_fwd_bwd, to64

pytestmark = pytest.mark.gpu

FULL_POINTS = [(N, d, dt) for dt in ("bf16", "fp32") for d in fa2_inputs.SWEEP_D for N in (128, 1024)]
LONG_POINTS = ([(8192, d, dt) for dt in ("bf16", "fp32") for d in (16, 64, 128)]
               + [(32768, 128, "bf16"), (32768, 128, "fp32")])


def _ids(points):
    return [f"n{N}-d{d}-{dt}" for N, d, dt in points]


@pytest.mark.parametrize("N,d,dtype", FULL_POINTS, ids=_ids(FULL_POINTS))
def test_sweep_point_full(oracle_mod, N, d, dtype):
    w = fa2_inputs.sweep_workload(N, d, dtype)
    inp = fa2_inputs.workload_inputs(w)
    got = gpu_fwd_bwd(inp, w.causal, w.scale)
    q, k, v, do = (to64(inp[n].float()) for n in ("q", "k", "v", "do"))
    o, lse = oracle_mod.forward(q, k, v, w.causal, w.scale)
    dq, dk, dv = oracle_mod.backward(q, k, v, do, w.causal, w.scale)
    for name, ref in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        e = assert_close(to64(got[name]), ref, dtype, name)
        print(f"ERR {w.name} all heads {name} max_abs {e:.3e}")


@pytest.mark.parametrize("N,d,dtype", LONG_POINTS, ids=_ids(LONG_POINTS))
def test_sweep_point_sampled(oracle_mod, N, d, dtype):
    w = fa2_inputs.sweep_workload(N, d, dtype)
    inp = fa2_inputs.workload_inputs(w)
    got = gpu_fwd_bwd(inp, w.causal, w.scale)
    heads = [w.H - 1] if N >= 32768 else [0, w.H - 1]
    for h in heads:
        rows = fa2_inputs.sample_rows(N, 128, seed=w.seed + h)
        q, k, v, do = (to64(inp[n][0, h].float()) for n in ("q", "k", "v", "do"))
        ref = oracle_mod.head_sampled(q, k, v, do, w.causal, w.scale, rows, rows)
        for name in ("o", "lse", "dq", "dk", "dv"):
            e = assert_close(to64(got[name][0, h][rows]), ref[name], dtype, f"{name}[head {h}]")
            print(f"ERR {w.name} head {h} sampled {name} max_abs {e:.3e}")
