"""Host logic of the multi-process benchmark on CPU: two `gloo` ranks.

Heads are independent in both passes, so N ranks each run the single-GPU path
on their own batch and exchange nothing on the data path; the only
inter-process steps are the barriers and the maximum of the per-rank device
times.  These tests run that logic with world size 2 on the CPU.
"""
import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import fa2_inputs  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, times, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        w = fa2_inputs.WORKLOADS["gpt2-small-b4h12-n512-d64"]
        inp = fa2_inputs.make_inputs(1, 2, 128, 16, "bf16", bench.rank_seed(w, rank))
        digest = torch.tensor([float(inp["q"].float().sum()), float(inp["do"].float().abs().sum())],
                              dtype=torch.float64)
        gathered = [torch.zeros_like(digest) for _ in range(WORLD)]
        dist.all_gather(gathered, digest)
        got = bench.max_over_ranks(dist, times[rank], dev)
        dist.barrier()
        torch.save({"gathered": [g.tolist() for g in gathered], "max": got},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_distinct_batches(tmp_path):
    # Rank 1 is slower on the first and third value, rank 0 on the second.
    times = [(10.0, 7.5, 3.0), (12.5, 6.0, 4.25)]
    mp.start_processes(_rank_main, args=(_free_port(), times, str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(WORLD)]
    want = [max(a, b) for a, b in zip(*times)]
    for r in range(WORLD):
        assert res[r]["max"] == want, r
    # Every rank sees the same gathered digests, and the two batches differ.
    assert res[0]["gathered"] == res[1]["gathered"]
    d0, d1 = res[0]["gathered"]
    assert d0 != d1


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(None, (1.5, 2, 3.25), torch.device("cpu")) == [1.5, 2.0, 3.25]


def test_whole_job_value_uses_slowest_rank():
    # Two ranks, 10 steps of 1e12 FLOP each per rank, slowest rank 20 ms in total.
    v = bench.whole_job_tflops(2, 1e12, 10, 20.0)
    assert v == pytest.approx(2 * 1e12 * 10 / 0.020 / 1e12)
    # Weak scaling: doubling the ranks at the same slowest time doubles the value.
    assert bench.whole_job_tflops(4, 1e12, 10, 20.0) == pytest.approx(2 * v)


def test_rank_seeds_differ_and_repeat():
    w = fa2_inputs.WORKLOADS["10b-b1h36-n4096-d128"]
    seeds = [bench.rank_seed(w, r) for r in range(8)]
    assert len(set(seeds)) == 8
    a = fa2_inputs.make_inputs(1, 1, 128, 16, "bf16", seeds[3])
    b = fa2_inputs.make_inputs(1, 1, 128, 16, "bf16", seeds[3])
    assert all(torch.equal(a[n], b[n]) for n in a)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(steps=3, warmup=3, gpus=2)
    assert bench.run_reference(args, fa2_inputs.WORKLOADS["10b-b1h36-n4096-d128"]) == 0
    assert capsys.readouterr().out == ""
