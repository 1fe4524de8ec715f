"""Benchmark: exact causal attention forward + backward on B200.

One step = the whole hot path on one batch: attn_fwd (O, LSE) then the
recompute backward (attn_bwd_preprocess, attn_bwd_main, attn_bwd_finalize),
on the fwd+bwd workload B=2, Hq=Hkv=32, L=4096, d=128, causal, synthetic
bf16 N(0,1) inputs.  Metric: algorithmic mask-adjusted TFLOP/s over fwd+bwd
(forward 4*d*visible_pairs*B*Hq; backward 2.5x that).

Multi-GPU (torchrun): the (batch, head) units are independent, so every rank
runs its own batch of the same workload with no collective on the data path
(weak scaling); the step time is the max over ranks.

`--impl reference` times the float64 CPU oracle (a slow, plain restatement of
the definition) on a bounded sample of the same workload instead.
"""

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, make_inputs  # noqa: E402

WORKLOAD = "mha_causal_fwdbwd"
METRIC = "attention TFLOP/s (bf16, mask-adjusted) fwd+bwd and % of B200 dense BF16 peak"
DOMINANT = "attn_bwd_main"
PROFILE = os.path.join(ROOT, "profiles", "attn_bwd_main_mha_causal_fwdbwd.md")
KERNEL_SRC = os.path.join(ROOT, "tiled_exact_attention_02_b200", "csrc", "attn_bwd.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=800)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--all-configs", action="store_true",
                    help="time attn_fwd and the backward on every workload (one JSON line each); not the bench line")
    ap.add_argument("--workload", default=None, help="with --all-configs: only this workload")
    ap.add_argument("--ring-blocks", type=int, default=0, metavar="N",
                    help="time one rank's block kernels of ring attention over N ranks (zigzag cut), all steps "
                         "run on this GPU without the exchange; not the bench line")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def roofline_peak(burst, sustained, region_ms, clk):
    """The measured GEMM peak that matches how the kernels were timed: the
    sustained figure (a seconds-long loop under the power cap) only when the
    timed region lasted a second or more and the clock sampler saw the power
    cap; otherwise the burst figure."""
    capped = bool(clk) and "sw_power_cap" in clk.get("reasons", [])
    if region_ms >= 1000.0 and capped:
        return sustained, "sustained (region >= 1 s under sw_power_cap)"
    return burst, "burst (region %.0f ms, %s)" % (region_ms, "power cap seen" if capped else "no power cap")


def profile_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    try:
        text = open(PROFILE).read()
        sha = hashlib.sha256(open(KERNEL_SRC, "rb").read()).hexdigest()[:16]
        m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
        m_b = re.search(r"dram_bytes_per_launch_full:\s*([0-9.eE+]+)", text)
        if m_sha and m_b and m_sha.group(1) == sha:
            return float(m_b.group(1))
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region.

    nvidia-smi needs a moment to start, so the sampler is started first and
    waits for its first sample; `mark()` brackets the timed region on the host
    clock and `stop()` keeps the samples whose timestamps fall inside it (the
    first one after it when the region is shorter than the sampling period)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
            return
        deadline = time.time() + 5.0
        while time.time() < deadline and not open(self.f.name).read().strip():
            time.sleep(0.05)

    def mark(self, start):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    @staticmethod
    def _when(stamp):
        from datetime import datetime
        try:
            return datetime.strptime(stamp.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.15)  # let a sample land after the region when it was shorter than the period
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = [[c.strip() for c in r.split(",")] for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        rows = [r for r in rows if len(r) >= 10]
        if not rows:
            return None
        timed = [r for r in rows if self.t0 is not None and self.t1 is not None
                 and (self._when(r[0]) or 0.0) >= self.t0 and (self._when(r[0]) or 0.0) <= self.t1]
        window = "timed region"
        if not timed:
            after = [r for r in rows if self.t0 is not None and (self._when(r[0]) or 0.0) >= self.t0]
            timed = after[:1] or rows[-1:]
            window = "first sample after the region started (region shorter than the 100 ms period)"
        sm = [float(r[2]) for r in timed]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in timed:
            for n, v in zip(names, r[6:10]):
                if v == "Active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(timed[0][3]),
                "power_w": statistics.median(float(r[4]) for r in timed),
                "samples": len(timed), "window": window, "reasons": sorted(reasons)}


def dist_setup(n_gpus, backend="nccl"):
    """Join the torchrun job (one process per GPU); returns (rank, world, local rank)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return rank, world, local


def rank_seed(w, rank):
    """Each rank draws its own batch of the workload (independent units)."""
    return w.seed + 1000 * rank


def max_over_ranks(x, world, device="cuda"):
    """The job's time is the slowest rank's."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, flops_per_rank_step, ms_per_step_max):
    """Whole-job TFLOP/s under weak scaling: every rank does one step's work."""
    return world * flops_per_rank_step / (ms_per_step_max * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


ROWS_PER_UNIT = 512  # CPU sample unit: 512 query rows of one head, fwd + their bwd contributions


def cpu_units(w):
    return [(b, h, r0) for b in range(w.B) for h in range(w.Hq) for r0 in range(0, w.Lq, ROWS_PER_UNIT)]


def unit_flops(w, r0):
    """Algorithmic fwd+bwd FLOPs of query rows [r0, r0 + ROWS_PER_UNIT) of one head."""
    pairs = 0
    for i in range(r0, min(w.Lq, r0 + ROWS_PER_UNIT)):
        hi = min(i + 1, w.Lk) if w.causal else w.Lk
        lo = max(0, i - w.window + 1) if w.window > 0 else 0
        pairs += max(0, hi - lo)
    return 3.5 * 4.0 * w.d * pairs


def oracle_sample(w, x, units):
    """Time the float64 oracle on sample units; returns (seconds, algorithmic flops)."""
    import oracle
    t0 = time.perf_counter()
    flops = 0.0
    for b, h, r0 in units:
        oracle.attn_row_block(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, w.window, b, h, r0,
                              min(w.Lq, r0 + ROWS_PER_UNIT))
        flops += unit_flops(w, r0)
    return time.perf_counter() - t0, flops


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[WORKLOAD]
    x = make_inputs(w)
    units = cpu_units(w)
    stride = 97  # walk the units in a fixed scattered order (mixes light and heavy causal rows)
    for i in range(args.warmup):
        oracle_sample(w, x, [units[(i * stride) % len(units)]])
    secs, flops = 0.0, 0.0
    for i in range(args.steps):
        s, f = oracle_sample(w, x, [units[((args.warmup + i) * stride) % len(units)]])
        secs += s
        flops += f
    value = flops / secs / 1e12
    cores = host_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.Lq, "d": w.d,
                   "causal": w.causal, "window": w.window,
                   "step_sample": f"{ROWS_PER_UNIT} query rows of one head, fwd + their bwd contributions"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} units of {ROWS_PER_UNIT} query rows x 1 head of {WORKLOAD}, "
                                   f"float64 numpy fwd+bwd, {secs:.1f} s"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def all_configs(args):
    """Forward and backward times of every workload on one GPU (CUDA-event
    medians; calls shorter than 1 ms timed in back-to-back groups), one JSON
    line each.  The
    backward runs with a dO drawn for the workload when it has none.  Inputs
    of the small case fit in L2; the others are larger than L2."""
    import numpy as np
    import torch
    import tiled_exact_attention_02_b200 as ta
    burst, sustained, hbm, peak_src = peaks()
    for name, w in WORKLOADS.items():
        if args.workload is not None and name != args.workload:
            continue
        x = make_inputs(w)
        dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = (dev(x[n]) for n in ("q", "k", "v"))
        do = dev(x["do"]) if "do" in x else torch.randn_like(q)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(ta.bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d), dtype=torch.uint8, device="cuda")

        def timed(fn, n):
            # Each sample brackets `rep` back-to-back calls (about 1 ms of work,
            # at most 10 calls), so for short kernels the host work of one call
            # overlaps the kernels of the one before it and the time is the
            # device's; the sample's mean per call, median over samples.
            fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            rep = max(1, min(10, int(1.0 / max(a.elapsed_time(b), 1e-3))))
            ts = []
            for it in range(n + 3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(rep):
                    fn()
                b.record()
                torch.cuda.synchronize()
                if it >= 3:
                    ts.append(a.elapsed_time(b) / rep)
            return statistics.median(ts)

        n = max(5, min(args.steps, 50))
        sb = w.sparse_block
        f_ms = timed(lambda: ta.fwd(q, k, v, o, lse, w.causal, w.window, w.scale, sparse_block=sb), n)
        ns = ta.lib.attn_fwd_split_default(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, ta._causal_code(w.causal), w.window)
        split = None
        if ns > 1 and not sb:
            sws = torch.empty(max(256, ta.lib.attn_fwd_split_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, ns)),
                              dtype=torch.uint8, device="cuda")
            s_ms = timed(lambda: ta.fwd_split(q, k, v, o, lse, ns, sws, w.causal, w.window, w.scale), n)
            split = {"n_split": ns, "fwd_ms": s_ms, "fwd_tflops": w.fwd_flops() / s_ms / 1e9}
        if sb:
            b_ms = timed(lambda: ta.bwd(q, k, v, o, lse, do, dq, dk, dv, ws, w.causal, w.window, w.scale,
                                        sparse_block=sb), n)
        else:
            b_ms = timed(lambda: ta.bwd_phases(q, k, v, o, lse, do, dq, dk, dv, ws, w.causal, w.window, w.scale), n)
        st, site = ta.device_error()
        if st != 0:
            raise SystemExit(f"device error {st} at site {site} on {name}")
        fwd_bytes = (q.numel() + k.numel() + v.numel() + o.numel()) * 2 + lse.numel() * 4
        print(json.dumps({
            "workload": name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.Lq, "d": w.d, "causal": w.causal,
            "window": w.window, "sparse_block": sb, "fwd_ms": f_ms, "fwd_tflops": w.fwd_flops() / f_ms / 1e9,
            "fwd_frac_spec_2250": w.fwd_flops() / f_ms / 1e9 / 2250.0,
            "fwd_algorithmic_GBs": fwd_bytes / f_ms / 1e6, "hbm_peak_GBs": hbm,
            "fwd_split": None if split is None else dict(split, fwd_algorithmic_GBs=fwd_bytes / split["fwd_ms"] / 1e6),
            "bwd_ms": b_ms, "bwd_tflops": w.bwd_flops() / b_ms / 1e9,
            "bwd_frac_spec_2250": w.bwd_flops() / b_ms / 1e9 / 2250.0,
            "peak_sustained_tflops": sustained, "peak_kind": peak_src}), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()


def ring_blocks(args):
    """One rank's compute in ring attention over N ranks (the zigzag cut gives
    every rank the same work): the forward and backward block calls of its N
    steps, timed with CUDA events on this GPU, on a causal sequence of 32768
    positions (B=1, Hq=32, Hkv=8, d=128).  The K/V chunks a rank would
    receive are taken from the full tensors, so no exchange is timed.  The
    monolithic forward and backward of the whole problem on this GPU, divided
    by N, is the comparison: it is what one GPU's share would cost without
    the cut into blocks."""
    import numpy as np
    import torch
    import tiled_exact_attention_02_b200 as ta
    from tiled_exact_attention_02_b200 import ring
    from synth import Workload
    N = args.ring_blocks
    w = Workload("ring_causal_32768", 1, 32, 8, 32768, 32768, 128, True, backward=True, seed=49)
    x = make_inputs(w)
    dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    full = {n: dev(x[n]) for n in ("q", "k", "v", "do")}
    sh = {n: [ring.shard(full[n], r, N, "zigzag") for r in range(N)] for n in full}
    ops = ring.CudaOps(ta.lib)
    r = 0  # every rank has the same work under the zigzag cut

    def timed(fn, reps=5):
        ts = []
        for it in range(reps + 2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if it >= 2:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    state = {}

    def fwd():
        f = ring.RingForwardRank(sh["q"][r], r, N, "zigzag", True, w.scale, ops)
        for t in range(N):
            src = (r - t) % N
            f.step(t, sh["k"][src], sh["v"][src])
        state["o"], state["lse"] = f.result()

    def bwd():
        bw = ring.RingBackwardRank(sh["q"][r], state["o"], state["lse"], sh["do"][r], r, N, "zigzag", True, w.scale,
                                   ops, k_like=sh["k"][r])
        acc = [torch.empty(sh["k"][r].shape, dtype=torch.float32, device="cuda") for _ in range(2)]
        for t in range(N):
            src = (r - t) % N
            bw.step(t, sh["k"][src], sh["v"][src], acc[0], acc[1])
        bw.dq()
        dk, dv = torch.empty_like(sh["k"][r]), torch.empty_like(sh["v"][r])
        ops.to_bf16(acc[0], dk)
        ops.to_bf16(acc[1], dv)

    f_ms = timed(fwd)
    b_ms = timed(bwd)
    q, k, v, do = (full[n] for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, True, 0, w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ta.bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d), dtype=torch.uint8, device="cuda")
    mf_ms = timed(lambda: ta.fwd(q, k, v, o, lse, True, 0, w.scale))
    mb_ms = timed(lambda: ta.bwd(q, k, v, o, lse, do, dq, dk, dv, ws, True, 0, w.scale))
    st, site = ta.device_error()
    if st != 0:
        raise SystemExit(f"device error {st} at site {site}")
    fl_f, fl_b = w.fwd_flops() / N, w.bwd_flops() / N
    print(json.dumps({
        "ring_blocks": N, "layout": "zigzag", "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.Lq,
        "d": w.d, "causal": True, "rank_chunks_rows": w.Lq // (2 * N),
        "rank_fwd_ms": f_ms, "rank_fwd_tflops": fl_f / f_ms / 1e9,
        "rank_bwd_ms": b_ms, "rank_bwd_tflops": fl_b / b_ms / 1e9,
        "monolithic_fwd_ms_over_N": mf_ms / N, "monolithic_bwd_ms_over_N": mb_ms / N,
        "block_efficiency_fwd": (mf_ms / N) / f_ms, "block_efficiency_bwd": (mb_ms / N) / b_ms}), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.all_configs:
        return all_configs(args)
    if args.ring_blocks:
        return ring_blocks(args)

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    import tiled_exact_attention_02_b200 as ta

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS[WORKLOAD]
    x = make_inputs(w, seed=rank_seed(w, rank))

    def dev_bf16(bits):
        import numpy as np
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, do = (dev_bf16(x[n]) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ta.bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    N_EV = 5  # fwd | pre | main | post boundaries
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(N_EV)] for _ in range(args.steps)]

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        ta.fwd(q, k, v, o, lse, w.causal, w.window, w.scale, stream)
        ta.bwd_phases(q, k, v, o, lse, do, dq, dk, dv, ws, w.causal, w.window, w.scale, stream,
                      between=(lambda i: evs[i + 1].record(stream)) if evs else None)

    for _ in range(max(3, args.warmup)):
        step()
    st, site = ta.device_error()
    if st != 0:
        raise SystemExit(f"device error {st} at site {site}")
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.mark(True)
    t_start.record(stream)
    for i in range(args.steps):
        step(events[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    barrier(world)
    clk = clocks.stop()
    st, site = ta.device_error()
    if st != 0:
        raise SystemExit(f"device error {st} at site {site}")
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world)
    ms_step = ms_total / args.steps
    flops_step = w.fwd_flops() + w.bwd_flops()
    value = job_throughput(world, flops_step, ms_step)

    names = ["attn_fwd", "attn_bwd_preprocess", "attn_bwd_main", "attn_bwd_finalize"]
    per = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in events) for j, n in enumerate(names)}
    burst, sustained, hbm, peak_src = peaks()
    main_ms = per[DOMINANT]
    achieved = w.bwd_flops() / (main_ms * 1e-3) / 1e12
    fwd_tf = w.fwd_flops() / (per["attn_fwd"] * 1e-3) / 1e12
    peak, peak_kind = roofline_peak(burst, sustained, ms_total, clk)

    # End to end through the C ABI's host-buffer call: attn_step_host copies
    # the pinned host inputs in, runs the step and copies every output (O,
    # LSE, dQ, dK, dV) back, overlapping the copies with the kernels chunk by
    # chunk.
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        ho, hlse, hdq, hdk, hdv = (pin(t) for t in (o, lse, dq, dk, dv))
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdq, hdk, hdv))
        hbuf = torch.empty(ta.step_host_buffer_size(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, True), dtype=torch.uint8,
                           device=dev)

        def e2e_step():
            ta.step_host(hq, hk, hv, ho, hlse, hbuf, do=hdo, dq=hdq, dk=hdk, dv=hdv, causal=w.causal,
                         window=w.window, scale=w.scale, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(b), world) / args.e2e_steps
        e2e = {"value": job_throughput(world, flops_step, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        xs = make_inputs(w)
        secs, fl, n = 0.0, 0.0, 0
        units = cpu_units(w)
        while secs < 12.0 and n < len(units):
            s, f = oracle_sample(w, xs, [units[(n * 97) % len(units)]])
            secs += s
            fl += f
            n += 1
        cpu = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
               "sample": f"{n} of {len(units)} units ({ROWS_PER_UNIT} query rows x 1 head) of {WORKLOAD}, "
                         f"float64 numpy fwd+bwd, {secs:.1f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.Lq, "d": w.d,
                   "causal": w.causal, "window": w.window, "global_batch": w.B * world,
                   "flops_per_step_per_gpu": flops_step, "parallelism": f"independent batches x{world}",
                   "l2": "inputs larger than L2 (Q,K,V,O,dO,dQ,dK,dV = 512 MB per GPU); no flush"},
        "frac_of_peak": {"spec_2250": value / world / 2250.0, f"{peak_src}_burst": value / world / burst,
                         f"{peak_src}_sustained": value / world / sustained},
        "kernels_ms": per,
        "fwd_tflops": fwd_tf,
        "roofline": {"kernel": DOMINANT, "bound": "tensor", "achieved": achieved, "peak": peak,
                     "peak_kind": f"{peak_src} bf16 {peak_kind}", "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
                     "traffic": profile_traffic()},
        "region": {"ms": ms_total, "sm_mhz_median": clk["sm_mhz"] if clk else None,
                   "kilocycles_per_step": ms_step * clk["sm_mhz"] if clk else None},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
