"""Benchmark: causal FlashAttention-2 forward + backward on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
fa2_forward (O, L) then fa2_backward (D / L pre-pass, dK/dV pass over key
tiles, dQ pass over query tiles), on the 10B-model head shape (B=1, H=36,
N=4096, d=128, bf16, causal) unless --workload names another.

Metric: attention TFLOP/s with causal FLOPs counted (forward 4*d*P_c,
backward 10*d*P_c, P_c = B*H*N(N+1)/2 unmasked query/key pairs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fa2|reference]
    python bench.py --table      # per-workload / sweep-point timing table

For N > 1 run under torchrun: each rank runs the same workload on its own
seeded batch (heads are independent; no collective on the data path), and the
reported value is the total FLOPs of all ranks over the slowest rank's time.
``--impl reference`` times the fp64 CPU oracle on the host instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import fa2_inputs  # noqa: E402

METRIC = "attention TFLOP/s (causal) fwd and fwd+bwd at 1 B200; % of bf16 tensor peak"
UNIT = "TFLOP/s"
SPEC_BF16_TFLOPS = 2250.0      # dense bf16 tensor peak of a B200 (spec sheet)
SPEC_TF32_TFLOPS = 1100.0      # dense TF32 tensor peak (half the 2.2 PF sparse figure)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of each
# bf16 d=128 kernel on the 10B head shape, from one ncu capture of the current
# kernel build; None where no capture of the current build exists.
FWD_TRAFFIC_BYTES = 207_431_168   # 185.2 MB read + 22.2 MB written
DKDV_TRAFFIC_BYTES = 201_089_792  # 153.4 MB read + 47.7 MB written (two-pass dK/dV pass)
DQ_TRAFFIC_BYTES = 177_845_760    # 154.3 MB read + 23.5 MB written (two-pass dQ pass)
FUSED_TRAFFIC_BYTES = None        # no capture of the one-pass backward's current build
TRAFFIC_WORKLOAD = "10b-b1h36-n4096-d128"


def causal_pairs(w) -> float:
    return w.B * w.H * w.N * (w.N + 1) / 2 if w.causal else w.B * w.H * w.N * w.N


def flops(w):
    pc = causal_pairs(w)
    return 4.0 * w.d * pc, 10.0 * w.d * pc


# Whether the library's default backward (fa2_backward, flags = 0) takes the
# one-pass form where it applies; mirrors kOnePassDefault in csrc/fa2_api.cu.
DEFAULT_BACKWARD_ONE_PASS = False


def one_pass(w) -> bool:
    """Whether the library's default backward takes its one-pass form on this
    (multi-head, no block mask) workload: 16-bit inputs and more than one key
    tile."""
    return DEFAULT_BACKWARD_ONE_PASS and w.dtype != "fp32" and w.N > 128


def single_tile_pairs(w) -> int:
    """Causal (query, key) pairs of the query tiles that see a single key tile
    (the first 128 rows of every causal head); their dQ comes from the
    query-tile pass in the one-pass form."""
    if not w.causal:
        return 0
    m = min(128, w.N)
    return w.B * w.H * m * (m + 1) // 2


def launches_per_step(w) -> int:
    """Library kernels one forward + backward launches."""
    if one_pass(w):
        return 1 + 1 + (1 if w.causal else 0) + 2    # fwd, pre, query-tile pass, key-tile pass, dQ rounding
    return 1 + 1 + 2                                    # fwd, pre, dQ pass, dK/dV pass


def block_sparse_pairs(mask, causal: bool, block: int = 128) -> int:
    """(query, key) pairs one head computes under a block mask of full
    block x block tiles: a full block off the diagonal, the lower triangle with
    the diagonal on it under the causal rule."""
    total = 0
    for i in range(mask.shape[0]):
        for j in range(mask.shape[1]):
            if not mask[i, j] or (causal and j > i):
                continue
            total += block * (block + 1) // 2 if (causal and i == j) else block * block
    return total


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {k: float(m[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the GPU legs
    run: through NVML (read-only queries, every 10 ms, on a host thread), or
    with `nvidia-smi -lms 100` where NVML is not importable.  Nothing here
    changes any GPU setting."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_s: float = 0.01):
        self.interval = interval_s
        self.samples = []          # (sm_mhz, max_mhz, reason bitmask)
        self.proc = None
        self.thread = None
        self.uuid = None
        try:
            u = str(torch.cuda.get_device_properties(device_index).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.target = self.uuid or str(device_index)

    def _nvml_loop(self, nv, handle):
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            self.stop.wait(self.interval)

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        try:
            import pynvml as nv
            nv.nvmlInit()
            handle = (nv.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                      else nv.nvmlDeviceGetHandleByIndex(int(self.target)))
            self.source = "nvml"
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, handle), daemon=True)
            self.thread.start()
        except Exception:
            self.source = "nvidia-smi"
            cmd = ["nvidia-smi", "-i", self.target, f"--query-gpu={self.FIELDS}",
                   "--format=csv,noheader,nounits", "-lms", "100"]
            try:
                self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                             stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
            time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for line in out.splitlines():
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm, mx = float(parts[0]), float(parts[1])
                except ValueError:
                    continue
                mask = 0
                for (nm, bit), val in zip(self.REASONS, parts[4:8]):
                    if val.lower() == "active":
                        mask |= bit
                self.samples.append((sm, mx, mask))
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": getattr(self, "source", None)}
        sm = sorted(s[0] for s in self.samples)
        reasons = sorted({nm for _, _, m in self.samples for nm, bit in self.REASONS if m & bit})
        return {"sm_mhz": sm[len(sm) // 2], "sm_min_mhz": sm[0], "sm_max_mhz": self.samples[-1][1],
                "reasons": reasons, "samples": len(sm), "source": self.source,
                "span": "warm-up, timed and end-to-end legs"}


# --------------------------------------------------------------------- CPU oracle

def oracle_step(w, sel):
    """fp64 oracle forward + backward on `sel` (a causal prefix of one head of
    the workload's inputs).  Returns (seconds, algorithmic FLOPs done)."""
    import oracle
    rows = sel["q"].shape[0]
    t0 = time.perf_counter()
    oracle.forward(sel["q"], sel["k"], sel["v"], w.causal, w.scale)
    oracle.backward(sel["q"], sel["k"], sel["v"], sel["do"], w.causal, w.scale)
    dt = time.perf_counter() - t0
    pairs = rows * (rows + 1) / 2 if w.causal else rows * rows
    return dt, 14.0 * w.d * pairs


def cpu_baseline(w, budget_s: float = 20.0):
    """The oracle as it stands, timed on the host cores over whole heads of the
    workload, head after head, until every head is done or `budget_s` seconds
    of oracle time have passed."""
    import oracle
    inp = fa2_inputs.workload_inputs(w)
    t, n = 0.0, 0
    for hh in range(w.heads):
        if t >= budget_s:
            break
        b, h = divmod(hh, w.H)
        sel = {k: inp[k][b, h].double().numpy() for k in ("q", "k", "v", "do")}
        t0 = time.perf_counter()
        oracle.forward(sel["q"], sel["k"], sel["v"], w.causal, w.scale)
        oracle.backward(sel["q"], sel["k"], sel["v"], sel["do"], w.causal, w.scale)
        t += time.perf_counter() - t0
        n += 1
    f = 14.0 * w.d * (w.N * (w.N + 1) / 2 if w.causal else w.N * w.N) * n
    return {"value": f / t / 1e12, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} of {w.heads} heads at full N={w.N}, d={w.d}, fwd+bwd, fp64",
            "seconds": round(t, 3)}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    # Bounded per-step sample: a causal prefix of one head, sized so the whole
    # run stays within a few minutes.
    steps = args.steps + args.warmup
    rows = min(w.N, max(256, int(w.N * math.sqrt(60.0 / max(steps, 1)))))
    rows = max(128, rows // 128 * 128)
    inp = fa2_inputs.workload_inputs(w)
    sel = {n: inp[n][0, 0, :rows].double().numpy() for n in ("q", "k", "v", "do")}
    del inp
    for _ in range(args.warmup):
        oracle_step(w, sel)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, f = oracle_step(w, sel)
        tot_t += dt
        tot_f += f
    value = tot_f / tot_t / 1e12
    sample = f"causal prefix of {rows} rows of head 0 (of {w.heads} heads, N={w.N}), fwd+bwd, fp64"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, n):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "dtype": w.dtype,
            "causal": w.causal, "scale": "1/sqrt(d)", "global_batch": w.B * n,
            "parallelism": f"replicas x{n} (independent heads, no collective)",
            "l2": "flushed between timed steps (256 MiB write)"}


# --------------------------------------------------------------------- table mode

def alg_bytes(w):
    """Algorithmic HBM bytes: forward reads Q, K, V and writes O and L; the
    backward reads Q, K, V, O, dO and L and writes dQ, dK, dV, with its two
    workspace vectors (D and L*log2(e)) counted once each."""
    es = 4 if w.dtype == "fp32" else 2
    t = w.B * w.H * w.N * w.d * es
    rows = w.B * w.H * w.N * 4
    return 4 * t + rows, 8 * t + 3 * rows


def run_table(args):
    """Times fa2_forward and fa2_backward on every model-table workload and a
    selection of sweep points (CUDA events, L2 flushed before each call) and
    prints one markdown table."""
    import causal_attention_fa2_b200 as fa2
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    meas = {"bf16": peaks["bf16_tflops"], "fp16": peaks["bf16_tflops"],
            "fp32": peaks["bf16_tflops"] * SPEC_TF32_TFLOPS / SPEC_BF16_TFLOPS}
    spec = {"bf16": SPEC_BF16_TFLOPS, "fp16": SPEC_BF16_TFLOPS, "fp32": SPEC_TF32_TFLOPS}
    points = list(fa2_inputs.WORKLOADS.values())
    w10 = fa2_inputs.WORKLOADS["10b-b1h36-n4096-d128"]
    points.append(fa2_inputs.Workload("10b-b1h36-n4096-d128-fp16", w10.B, w10.H, w10.N, w10.d, "fp16", w10.seed))
    # Grouped-query points: (workload, key/value heads).
    gqa = {"10b-b1h36-n4096-d128-gqa-kv4": 4, "10b-b1h36-n4096-d128-mqa": 1}
    for name in gqa:
        points.append(fa2_inputs.Workload(name, w10.B, w10.H, w10.N, w10.d, "bf16", w10.seed))
    # Block-sparse points: block masks over the 32 x 32 tiles of 128 rows
    # (a band of 4 tiles: each query tile sees itself and the 3 before it;
    # and a seeded random mask of density 1/2 that keeps the diagonal).
    nt = w10.N // 128
    band = np.zeros((nt, nt), dtype=np.uint8)
    for i in range(nt):
        band[i, max(0, i - 3):i + 1] = 1
    rnd = (np.random.default_rng(7).random((nt, nt)) < 0.5).astype(np.uint8)
    np.fill_diagonal(rnd, 1)
    sparse = {"10b-b1h36-n4096-d128-band4": band, "10b-b1h36-n4096-d128-bs50": rnd}
    for name in sparse:
        points.append(fa2_inputs.Workload(name, w10.B, w10.H, w10.N, w10.d, "bf16", w10.seed))
    points += [fa2_inputs.sweep_workload(N, d, dt) for dt in ("bf16", "fp32") for d in fa2_inputs.SWEEP_D
               for N in (128, 512, 1024, 4096, 8192, 16384, 32768)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    print(f"peaks: bf16 {meas['bf16']:.1f} TFLOP/s ({peak_src}); TF32 {meas['fp32']:.1f} "
          f"(bf16 x 1100/2250); HBM {peaks['hbm_gbs']:.1f} GB/s")
    print("| workload | dtype | fwd ms | fwd TFLOP/s | fwd % spec / % meas | fwd GB/s | bwd ms | "
          "bwd TFLOP/s | bwd % spec / % meas | bwd GB/s |")
    print("|---|---|---|---|---|---|---|---|---|---|")
    for w in points:
        g = torch.Generator(device="cpu")
        g.manual_seed(w.seed)
        dt = fa2_inputs.DTYPES[w.dtype]
        h_kv = gqa.get(w.name, w.H)
        q, k, v, do = (torch.randn((w.B, h, w.N, w.d), generator=g).to(dt).to(dev)
                       for h in (w.H, h_kv, h_kv, w.H))
        o, lse = fa2.forward(q, k, v, causal=w.causal, scale=w.scale,
                             block_mask=(torch.from_numpy(sparse[w.name]).to(dev) if w.name in sparse else None))
        ws = torch.empty(fa2.backward_workspace_bytes(w.B, w.H, w.N, w.d, q.dtype, h_kv), dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        f_fwd, f_bwd = flops(w)
        bm = None
        if w.name in sparse:
            bm = torch.from_numpy(sparse[w.name]).to(dev)
            pc = w.B * w.H * block_sparse_pairs(sparse[w.name], w.causal)
            f_fwd, f_bwd = 4.0 * w.d * pc, 10.0 * w.d * pc
        b_fwd, b_bwd = alg_bytes(w)
        reps = max(3, min(args.steps, 20))
        tf, tb = [], []
        for i in range(reps + 3):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record()
            fa2.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, block_mask=bm)
            e[1].record()
            flush.zero_()
            e2 = torch.cuda.Event(enable_timing=True)
            e2.record()
            fa2.backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, workspace=ws,
                         dq=dq, dk=dk, dv=dv, block_mask=bm)
            e[2].record()
            torch.cuda.synchronize()
            if i >= 3:
                tf.append(e[0].elapsed_time(e[1]))
                tb.append(e2.elapsed_time(e[2]))
        mf, mb = sorted(tf)[len(tf) // 2], sorted(tb)[len(tb) // 2]
        tff, tfb = f_fwd / mf / 1e9, f_bwd / mb / 1e9
        print(f"| {w.name} | {w.dtype} | {mf:.4f} | {tff:.1f} | {100 * tff / spec[w.dtype]:.1f} / "
              f"{100 * tff / meas[w.dtype]:.1f} | {b_fwd / mf / 1e6:.0f} | {mb:.4f} | {tfb:.1f} | "
              f"{100 * tfb / spec[w.dtype]:.1f} / {100 * tfb / meas[w.dtype]:.1f} | {b_bwd / mb / 1e6:.0f} |",
              flush=True)
        del q, k, v, do, o, lse, ws, dq, dk, dv
    status = fa2.last_device_status()
    if status != 0:
        raise SystemExit(f"device status after timing: {fa2.status_string(status)}")
    return 0


# --------------------------------------------------------------------- ranks

def rank_seed(w, rank: int) -> int:
    """Seed of a rank's own batch: every rank draws a different batch of the
    same shape (weak scaling; heads are independent, so ranks never exchange
    data)."""
    return w.seed + rank


def max_over_ranks(dist, values, device):
    """Element-wise maximum of `values` over all ranks, returned on every rank;
    the values unchanged when there is one process (`dist` None)."""
    if dist is None:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(world: int, flops_per_rank_step: float, steps: int, ms: float) -> float:
    """Work of all ranks over `steps` steps divided by the slowest rank's time."""
    return world * flops_per_rank_step * steps / (ms * 1e-3) / 1e12


# --------------------------------------------------------------------- GPU arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fa2", choices=["fa2", "reference"])
    ap.add_argument("--workload", default="10b-b1h36-n4096-d128")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--table", action="store_true",
                    help="time every model-table workload and sweep point; print a table")
    args = ap.parse_args()
    if args.table:
        return run_table(args)
    w = fa2_inputs.workload_by_name(args.workload)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, w)

    import causal_attention_fa2_b200 as fa2

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    # Inputs: each rank its own seeded batch (weak scaling).
    inp = fa2_inputs.make_inputs(w.B, w.H, w.N, w.d, w.dtype, rank_seed(w, rank))
    host = {n: t.pin_memory() for n, t in inp.items()}
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa2.backward_workspace_bytes(w.B, w.H, w.N, w.d, q.dtype),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    f_fwd, f_bwd = flops(w)

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        fa2.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)
        fa2.backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, workspace=ws,
                     dq=dq, dk=dk, dv=dv, events=None if evs is None else evs[1:5])
        if evs is not None:
            evs[5].record()

    # Clocks are sampled from the first warm-up step to the end of the
    # end-to-end leg (the timed region itself is a few tens of milliseconds).
    sampler = ClockSampler(local)
    sampler.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for e in evs:          # materialise the event handles before handing them out
        for x in e:
            x.record()
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()                          # evict the previous step from L2
        step(evs[i])
    torch.cuda.synchronize()
    barrier()
    t_fwd = [e[0].elapsed_time(e[1]) for e in evs]          # forward kernel
    t_bwd = [e[1].elapsed_time(e[5]) for e in evs]          # whole backward call
    t_pre = [e[1].elapsed_time(e[2]) for e in evs]          # D / L pre-pass
    t_dq = [e[2].elapsed_time(e[3]) for e in evs]           # query-tile pass
    t_dkdv = [e[3].elapsed_time(e[4]) for e in evs]         # key-tile pass
    t_fin = [e[4].elapsed_time(e[5]) for e in evs]          # dQ rounding (one-pass form)
    t_step = [a + b for a, b in zip(t_fwd, t_bwd)]
    total_ms = sum(t_step)
    fwd_ms, bwd_ms = sum(t_fwd), sum(t_bwd)
    total_ms, fwd_ms, bwd_ms = max_over_ranks(dist, (total_ms, fwd_ms, bwd_ms), dev)
    status = fa2.last_device_status()
    if status != 0:
        raise SystemExit(f"device status after timing: {fa2.status_string(status)}")

    # ---------------- end to end through the public API with host buffers
    # Every step copies its inputs from pinned host memory, runs forward and
    # backward, and copies its results back.  Three streams and two device
    # buffer sets let step i's input copies and step i-1's output copies run
    # while step i-1's / step i's kernels do: a set's inputs are overwritten
    # only after the kernels of the step two back have read them, and its
    # outputs only after their copy to the host has finished.
    out_names = ("o", "lse", "dq", "dk", "dv")
    out_host = {n: torch.empty_like(t if n != "lse" else lse, device="cpu").pin_memory()
                for n, t in (("o", q), ("lse", lse), ("dq", q), ("dk", q), ("dv", q))}
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v", "do"))
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    K_e2e = max(3, min(K, 50))
    sets = [dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_run(n_steps, start=None, end=None):
        ev_in = [torch.cuda.Event() for _ in range(n_steps)]
        ev_cmp = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        if start is not None:
            start.record(s_in)
        for i in range(n_steps):
            b = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])
                for n in ("q", "k", "v", "do"):
                    b[n].copy_(host[n], non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    s_cmp.wait_event(ev_out[i - 2])
                fa2.forward(b["q"], b["k"], b["v"], causal=w.causal, scale=w.scale,
                            out=b["o"], lse=b["lse"])
                fa2.backward(b["q"], b["k"], b["v"], b["o"], b["lse"], b["do"], causal=w.causal,
                             scale=w.scale, workspace=ws, dq=b["dq"], dk=b["dk"], dv=b["dv"])
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                for n in out_names:
                    out_host[n].copy_(b[n], non_blocking=True)
                ev_out[i].record(s_out)
        if end is not None:
            end.record(s_out)

    torch.cuda.synchronize()
    ref_host = {n: sets[0][n].cpu() for n in out_names}     # the device-timed loop's results
    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(K_e2e, e_start, e_end)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    # The last step's results, read back on the host, must be the bits the
    # device-timed loop produced from the same inputs -- except dQ, whose
    # one-pass form sums key tiles by fp32 reduce-add in an order that can
    # change between runs: it must agree to within its 16-bit rounding.
    for n in out_names:
        same = (torch.allclose(out_host[n].float(), ref_host[n].float(), atol=1e-3, rtol=1e-2)
                if n == "dq" else torch.equal(out_host[n], ref_host[n]))
        if not same:
            raise SystemExit(f"end-to-end leg: host copy of {n} differs from the device result")
    sampler.__exit__(None, None, None)
    (e2e_ms,) = max_over_ranks(dist, (e2e_ms,), dev)
    barrier()

    if rank == 0:
        peaks, peak_src = load_peaks()
        value = whole_job_tflops(world, f_fwd + f_bwd, K, total_ms)
        fwd_tf = whole_job_tflops(world, f_fwd, K, fwd_ms)
        bwd_tf = whole_job_tflops(world, f_bwd, K, bwd_ms)
        avg_fwd = sum(t_fwd) / K
        avg_dkdv = sum(t_dkdv) / K
        avg_dq = sum(t_dq) / K
        # Dominant kernel: the one with the largest share of the step, with its
        # algorithmic FLOPs.  One-pass form: the key-tile pass does S, dP, dV,
        # dK on every causal pair and dQ on all but the single-tile pairs
        # (10*d*P_c - 2*d*single); the query-tile pass run on the single-tile
        # query tiles counts their dQ only (2*d*single).  Two-pass form: dK/dV
        # pass 8*d*P_c; dQ pass 2*d*P_c (its recomputed S and dP are not
        # algorithmic work).
        pc4 = f_fwd / 4.0
        single = single_tile_pairs(w)
        onep = one_pass(w)
        if onep:
            names = (f"fa2_fwd2_kernel<{w.dtype},d={w.d}>", f"fa2_bwd_fused_kernel<{w.dtype},d={w.d}>",
                     f"fa2_bwd_dq_kernel<{w.dtype},d={w.d}> (single-tile query tiles)")
            traffic = ((FWD_TRAFFIC_BYTES, FUSED_TRAFFIC_BYTES, None)
                       if w.name == TRAFFIC_WORKLOAD else (None, None, None))
            flops_k = (10 * pc4 - 2 * w.d * single, 2 * w.d * single)
        elif w.dtype != "fp32":
            names = (f"fa2_fwd2_kernel<{w.dtype},d={w.d}>", f"fa2_bwd_dkdv_kernel<{w.dtype},d={w.d}>",
                     f"fa2_bwd_dq_kernel<{w.dtype},d={w.d}>")
            traffic = ((FWD_TRAFFIC_BYTES, DKDV_TRAFFIC_BYTES, DQ_TRAFFIC_BYTES)
                       if w.name == TRAFFIC_WORKLOAD else (None, None, None))
            flops_k = (8 * pc4, 2 * pc4)
        else:
            names = (f"fa2_fwd_kernel<fp32,d={w.d}>", f"fa2_bwd32_dkdv_kernel<d={w.d}>",
                     f"fa2_bwd32_dq_kernel<d={w.d}>")
            traffic = (None, None, None)
            flops_k = (8 * pc4, 2 * pc4)
        cands = [(avg_fwd, names[0], f_fwd, traffic[0]),
                 (avg_dkdv, names[1], flops_k[0], traffic[1]),
                 (avg_dq, names[2], flops_k[1], traffic[2])]
        kms, kname, kflops, ktraffic = max(cands, key=lambda c: c[0])
        achieved = kflops / (kms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": config_of(w, world),
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "fwd_frac_of_spec_bf16": fwd_tf / world / SPEC_BF16_TFLOPS,
            "bwd_frac_of_spec_bf16": bwd_tf / world / SPEC_BF16_TFLOPS,
            "fwd_frac_of_measured_bf16": fwd_tf / world / peaks["bf16_tflops"],
            "bwd_frac_of_measured_bf16": bwd_tf / world / peaks["bf16_tflops"],
            "ms": {"fwd": avg_fwd, "bwd_pre": sum(t_pre) / K,
                   "bwd_query_tile_pass": avg_dq, "bwd_key_tile_pass": avg_dkdv,
                   "bwd_dq_round": sum(t_fin) / K},
            "backward_form": "one pass (key tiles outer, dQ by fp32 reduce-add)" if onep
                             else "two passes (Algorithm 2)",
            "e2e": {"value": whole_job_tflops(world, f_fwd + f_bwd, K_e2e, e2e_ms),
                    "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": K_e2e},
            "gpu_launches": launches_per_step(w) * K,
            "roofline": {"bound": "tensor", "kernel": kname, "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": UNIT,
                         "frac": achieved / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16 dense (burst)",
                         "flops_per_launch": kflops, "ms_per_launch": kms,
                         "traffic": ktraffic},
            "clocks": sampler.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            oracle.build()
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
