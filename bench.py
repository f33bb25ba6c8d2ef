#!/usr/bin/env python
"""Benchmark of the ring attention hot path on B200.

Headline: causal-adjusted attention TFLOPS of the ring forward on the Llama-3-8B
layer shape at 32k tokens (B=1, 32 query heads over 8 KV heads, D=128, P=8
virtual ranks in zigzag order, causal, bf16 in / fp32 accumulate), as a
fraction of the measured dense BF16 peak. One step = one forward launch over
one batch of synthetic input already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own replica (weak scaling, no exchange: the
ring is simulated on each GPU); the time is the max over ranks. Also reported:
e2e (host buffers, copies inside the timed region), the roofline of the
forward kernel, the CPU oracle as a baseline, sampled SM clocks, and the
other hot-path kernels (Ulysses permute, backward) as extra entries.
`--impl reference` times the fp64 CPU oracle on bounded samples of the same
workload and prints the same line with "impl": "reference".
"""
import argparse
import faulthandler
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
faulthandler.enable()

METRIC = "causal-adj attention TFLOPS, % of B200 BF16 peak (S=32k GQA ring fwd)"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--only", choices=["all", "fwd", "permute", "bwd", "window", "packed",
                                      "layout", "allgather", "steps", "bwdsteps", "exchange"],
                   default="all",
                   help="restrict to one kernel (used for profiling runs)")
    p.add_argument("--skip-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--skip-e2e", action="store_true")
    p.add_argument("--bwd-heads", type=int, default=None,
                   help="heads of the backward case (default: the workload's; smaller for profiling)")
    args = p.parse_args()
    if args.warmup < 3 and args.only == "all":
        p.error("at least 3 warm-up steps")
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(summary_name, sources):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith(" "):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_sha256") != source_digest(sources):
            return None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index, period_s=0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            want = (getattr(props, "pci_domain_id", None), getattr(props, "pci_bus_id", None),
                    getattr(props, "pci_device_id", None))
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                info = pynvml.nvmlDeviceGetPciInfo(h)
                if (int(info.domain), int(info.bus), int(info.device)) == want:
                    self.handle = h
                    break
            if self.handle is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
                self.nvml = pynvml
        except Exception:
            self.handle = None

    def _run(self):
        nv = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                bits = int(get_reasons(self.handle))
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.handle is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def time_on_stream(fn, steps, stream):
    """Device time (ms) of `steps` calls of fn, with CUDA events on `stream`."""
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, nrows_per_head, seed):
    """Times the fp64 oracle on nrows_per_head seeded query rows of every head
    of workload w. Returns (seconds, algorithmic FLOPs of the sample, threads)."""
    import numpy as np
    import oracle
    from ring_ulysses_sequence_b200.synth import make_inputs
    if not hasattr(oracle_sample, "_cache"):
        oracle_sample._cache = {}
    if w.name not in oracle_sample._cache:
        q, k, v = make_inputs(w, with_dout=False)
        oracle_sample._cache[w.name] = (q.float(), k.float(), v.float())
    q, k, v = oracle_sample._cache[w.name]
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(w.S, size=nrows_per_head, replace=False))
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, w.causal, rows=rows)
    dt = time.perf_counter() - t0
    keys = (rows + 1) if w.causal else np.full(len(rows), w.S)
    flops = float(4.0 * w.D * keys.sum() * w.B * w.H)
    return dt, flops, oracle.num_threads()


def calibrate_rows(w, target_s, seed=0, hi=4096):
    """Rows per head that make one oracle sample take about target_s seconds
    (two-point fit: the per-call fixed cost is separated from the per-row cost).
    Both fit points keep every oracle thread busy (the oracle hands rows out in
    chunks of 4), else the per-row cost would come out too small."""
    import oracle
    lo = max(64, 8 * oracle.num_threads())
    t_lo, _, _ = oracle_sample(w, lo, seed)
    t_hi, _, _ = oracle_sample(w, 4 * lo, seed + 1)
    per_row = max((t_hi - t_lo) / (3 * lo), 1e-6)
    fixed = max(t_lo - lo * per_row, 0.0)
    return int(max(16, min(hi, (target_s - fixed) / per_row)))


def cpu_baseline(w, target_s=15.0):
    n = calibrate_rows(w, target_s)
    dt, flops, threads = oracle_sample(w, n, seed=12345)
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{n} seeded query rows of each of the {w.B * w.H} heads "
                      f"(all their visible keys), fp64, {dt:.1f} s"}


def run_reference(args):
    from ring_ulysses_sequence_b200 import multi
    from ring_ulysses_sequence_b200.synth import BENCH_WORKLOAD, WORKLOADS
    rank, world, _ = multi.env_ranks()
    if rank != 0:
        return
    w = WORKLOADS[BENCH_WORKLOAD]
    per_step = max(0.3, min(10.0, 150.0 / (args.steps + args.warmup)))
    n = calibrate_rows(w, per_step)
    for i in range(args.warmup):
        oracle_sample(w, n, seed=i)
    tot_s, tot_f, threads = 0.0, 0.0, 1
    for i in range(args.steps):
        dt, fl, threads = oracle_sample(w, n, seed=1000 + i)
        tot_s += dt
        tot_f += fl
    value = tot_f / tot_s / 1e12
    sample = (f"per step {n} seeded query rows of each of the {w.B * w.H} heads "
              f"(all their visible keys), fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w):
    """The workload's config (the same for the GPU arm and the reference arm)."""
    eb = 2 if "bf16" in w.name else 4
    bytes_in = (w.B * w.H + 2 * w.B * w.Hkv) * w.S * w.D * eb
    bytes_out = w.B * w.H * w.S * (w.D * eb + 4)
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "S": w.S, "D": w.D, "P": w.P,
            "order": w.order, "causal": w.causal, "global_batch": w.B, "seq_len": w.S,
            "parallelism": f"ring P={w.P} simulated per GPU",
            "l2": f"inputs {bytes_in / 1e6:.0f} MB + outputs {bytes_out / 1e6:.0f} MB "
                  f"> {L2_BYTES >> 20} MiB L2 (no flush)"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def bench_forward(w, args, dev, stream):
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import multi
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q = (torch.randn((w.B, w.H, w.S, w.D), generator=g, device=dev) * w.input_scale).to(w.dtype)
    k = (torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, device=dev) * w.input_scale).to(w.dtype)
    v = (torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, device=dev) * w.input_scale).to(w.dtype)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)

    def step():
        rm.ring_attn_fwd(q, k, v, w.P, w.causal, w.order, out=o, lse=lse, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    multi.barrier(dev)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    with sampler:
        ms = time_on_stream(step, args.steps, stream)
    torch.cuda.synchronize()
    multi.barrier(dev)
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the forward benchmark")
    ms_max = multi.max_over_ranks(ms, dev)
    bytes_in = sum(t.numel() * t.element_size() for t in (q, k, v))
    bytes_out = o.numel() * o.element_size() + lse.numel() * 4
    res = {"ms_total": ms_max, "launches": args.steps, "clocks": sampler.summary(),
           "bytes_in": bytes_in, "bytes_out": bytes_out}

    if not args.skip_e2e:
        res["e2e"] = bench_forward_e2e(w, args, dev, stream, (q, k, v, o, lse))
    return res


def bench_forward_e2e(w, args, dev, stream, tensors):
    """End to end through the public API: every step copies its q, k, v from
    pinned host memory, runs the forward and copies O and LSE back to pinned
    host memory. Two device buffer sets and three streams let the copy in of
    step i + 1 and the copy out of step i - 1 run on the copy engines while the
    forward of step i runs; each step still moves all of its own bytes inside
    the timed region."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import multi
    q0, k0, v0, o0, lse0 = tensors
    hq, hk, hv = (t.cpu().pin_memory() for t in (q0, k0, v0))
    ho = torch.empty(o0.shape, dtype=o0.dtype, pin_memory=True)
    hl = torch.empty(lse0.shape, dtype=lse0.dtype, pin_memory=True)
    bufs = [(q0, k0, v0, o0, lse0)] + [tuple(torch.empty_like(t) for t in tensors)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        q, k, v, o, lse = bufs[b]
        if used[b]:
            s_in.wait_event(ev_fwd[b])     # the forward of step i - 2 has read q, k, v
        with torch.cuda.stream(s_in):
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if used[b]:
            stream.wait_event(ev_out[b])   # step i - 2's O, LSE are out of this buffer
        rm.ring_attn_fwd(q, k, v, w.P, w.causal, w.order, out=o, lse=lse, stream=stream)
        ev_fwd[b].record(stream)
        s_out.wait_event(ev_fwd[b])
        with torch.cuda.stream(s_out):
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    e2e_steps = max(4, min(args.steps, 50))
    for i in range(2):  # warm-up
        e2e_step(i)
    torch.cuda.synchronize()
    multi.barrier(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    end.record(s_out)
    end.synchronize()
    ms = start.elapsed_time(end)
    multi.barrier(dev)
    bytes_in = sum(t.numel() * t.element_size() for t in (q0, k0, v0))
    bytes_out = o0.numel() * o0.element_size() + lse0.numel() * 4
    return {"ms_per_step": multi.max_over_ranks(ms, dev) / e2e_steps, "steps": e2e_steps,
            "h2d": bytes_in, "d2h": bytes_out}


def bench_permute(args, dev, stream):
    """Fused Q/K/V Ulysses permute (sequence- to head-sharded), 131072 tokens."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS
    w = WORKLOADS["usp_fwd_bf16_S128k_u4r4"]
    U, R = w.ulysses, w.P
    q = torch.randn((w.B, w.S, w.H, w.D), device=dev).to(w.dtype)
    k = torch.randn((w.B, w.S, w.Hkv, w.D), device=dev).to(w.dtype)
    v = torch.randn((w.B, w.S, w.Hkv, w.D), device=dev).to(w.dtype)
    outs = [torch.empty((w.B, w.H, w.S, w.D), device=dev, dtype=w.dtype),
            torch.empty((w.B, w.Hkv, w.S, w.D), device=dev, dtype=w.dtype),
            torch.empty((w.B, w.Hkv, w.S, w.D), device=dev, dtype=w.dtype)]

    def step():
        rm.ulysses_permute_qkv(q, k, v, U, R, "seq_to_head", outs=outs, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 100))
    ms = time_on_stream(step, steps, stream) / steps
    moved = 2 * sum(t.numel() * t.element_size() for t in (q, k, v))  # read + write
    return {"workload": w.name, "ms_per_launch": ms, "bytes_per_launch": moved,
            "gbs": moved / ms / 1e6, "launches": steps + max(3, args.warmup)}


def bench_layout(args, dev, stream):
    """The HBM-bound helpers on the bench workload's tensors: natural -> rank-major
    reorder of Q (bf16), and the standalone (O, LSE) merge of one fp32 partial
    into a running pair for every query row."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS, BENCH_WORKLOAD
    w = WORKLOADS[BENCH_WORKLOAD]
    q = torch.randn((w.B, w.H, w.S, w.D), device=dev).to(w.dtype)
    q_rm = torch.empty_like(q)
    rows = w.B * w.H * w.S
    o_acc = torch.randn((rows, w.D), device=dev)
    o_part = torch.randn((rows, w.D), device=dev)
    l_acc = torch.randn(rows, device=dev)
    l_part = torch.randn(rows, device=dev)
    steps = max(5, min(args.steps, 50))
    out = {}
    for name, fn, moved in (
            ("seq_reorder", lambda: rm.seq_reorder(q, w.P, w.order, "to_rank_major", out=q_rm,
                                                   stream=stream),
             2 * q.numel() * q.element_size()),
            ("lse_merge", lambda: rm.lse_merge_(o_acc, l_acc, o_part, l_part, stream=stream),
             (3 * rows * w.D + 3 * rows) * 4)):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        ms = time_on_stream(fn, steps, stream) / steps
        out[name] = {"ms": ms, "bytes_per_launch": moved, "gbs": moved / ms / 1e6}
    return out


def bench_allgather(args, dev, stream):
    """The all-gather alternative to the ring on the bench workload: gather K/V
    into natural order (two reorders, the one-device form of the collective),
    then one attention pass. Timed whole and attention alone; the per-rank K/V
    residency of both designs in a real P-rank run is reported beside it."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS, BENCH_WORKLOAD
    w = WORKLOADS[BENCH_WORKLOAD]
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q, k, v = ((torch.randn(s, generator=g, device=dev) * w.input_scale).to(w.dtype)
               for s in [(w.B, w.H, w.S, w.D), (w.B, w.Hkv, w.S, w.D), (w.B, w.Hkv, w.S, w.D)])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    kv_all = [torch.empty_like(k), torch.empty_like(v)]

    def gather():
        rm.allgather_kv(k, v, w.P, w.order, outs=kv_all, stream=stream)

    def attend():
        rm.allgather_attn_fwd(q, kv_all[0], kv_all[1], w.P, w.causal, w.order, out=o, lse=lse,
                              stream=stream)

    def step():
        gather()
        attend()

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 100))
    ms = time_on_stream(step, steps, stream) / steps
    ms_attn = time_on_stream(attend, steps, stream) / steps
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the all-gather benchmark")
    kv_block = 2 * (w.S // w.P) * w.B * w.Hkv * w.D * k.element_size()  # K + V of one rank
    return {"workload": w.name, "ms_per_step": ms, "ms_attention": ms_attn,
            "tflops": w.fwd_flops() / ms / 1e9, "tflops_attention": w.fwd_flops() / ms_attn / 1e9,
            "flops_per_launch": w.fwd_flops(),
            "kv_bytes_per_rank": {"ring": 2 * kv_block, "allgather": w.P * kv_block}}


def bench_steps(args, dev, stream):
    """The bench workload as the ranks of a multi-device ring would run it, all
    on this device: for each of the P ranks, P launches of
    rm_ring_attn_fwd_step (its queries against one owner block) and P
    rm_lse_merge folds. The block exchange itself is not part of this (one
    device); the figure is the cost of splitting the fused ring into steps."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS, BENCH_WORKLOAD
    w = WORKLOADS[BENCH_WORKLOAD]
    L = w.S // w.P
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q, k, v = ((torch.randn(s, generator=g, device=dev) * w.input_scale).to(w.dtype)
               for s in [(w.P, w.B, w.H, L, w.D), (w.P, w.B, w.Hkv, L, w.D),
                         (w.P, w.B, w.Hkv, L, w.D)])
    o_acc = torch.empty((w.P, w.B, w.H, L, w.D), dtype=torch.float32, device=dev)
    l_acc = torch.empty((w.P, w.B, w.H, L), dtype=torch.float32, device=dev)
    o_p = torch.empty((w.B, w.H, L, w.D), dtype=torch.float32, device=dev)
    l_p = torch.empty((w.B, w.H, L), dtype=torch.float32, device=dev)

    def reset():
        with torch.cuda.stream(stream):
            o_acc.zero_()
            l_acc.fill_(float("-inf"))

    def step():  # the fused call: each step folds straight into the running pair
        reset()
        for rank in range(w.P):
            for t in range(w.P):
                owner = (rank - t) % w.P
                rm.ring_attn_fwd_step_merge(q[rank], k[owner], v[owner], o_acc[rank],
                                            l_acc[rank], w.P, rank, owner, w.causal, w.order,
                                            stream=stream)

    def step_two_calls():  # the partial written out, then merged by rm_lse_merge
        reset()
        for rank in range(w.P):
            for t in range(w.P):
                owner = (rank - t) % w.P
                rm.ring_attn_fwd_step(q[rank], k[owner], v[owner], w.P, rank, owner, w.causal,
                                      w.order, out=o_p, lse=l_p, stream=stream)
                rm.lse_merge_(o_acc[rank], l_acc[rank], o_p, l_p, stream=stream)

    for fn in (step, step_two_calls):
        for _ in range(max(3, args.warmup)):
            fn()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 20))
    ms = time_on_stream(step, steps, stream) / steps
    ms2 = time_on_stream(step_two_calls, steps, stream) / steps
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the step benchmark")
    return {"workload": w.name, "ms_per_step": ms, "tflops": w.fwd_flops() / ms / 1e9,
            "launches_per_step": w.P * w.P + 2, "flops_per_step": w.fwd_flops(),
            "ms_per_step_two_calls": ms2, "tflops_two_calls": w.fwd_flops() / ms2 / 1e9}


def bench_bwd_steps(args, dev, stream):
    """The backward of the bench workload as the ranks of a multi-device ring
    would run it, all on this device: per rank one rm_ring_attn_bwd_delta, and
    P rm_ring_attn_bwd_step launches in the reverse ring's schedule (dQ
    accumulating on the rank, dK/dV on the block). No exchange (one device)."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS, BENCH_WORKLOAD
    w = WORKLOADS[BENCH_WORKLOAD]
    L = w.S // w.P
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q, k, v, do = ((torch.randn(s, generator=g, device=dev) * w.input_scale).to(w.dtype)
                   for s in [(w.P, w.B, w.H, L, w.D), (w.P, w.B, w.Hkv, L, w.D),
                             (w.P, w.B, w.Hkv, L, w.D), (w.P, w.B, w.H, L, w.D)])
    qr, kr, vr = (x.permute(1, 2, 0, 3, 4).reshape(w.B, x.shape[2], w.S, w.D).contiguous()
                  for x in (q, k, v))
    o, lse = rm.ring_attn_fwd(qr, kr, vr, w.P, w.causal, w.order, stream=stream)
    o = o.reshape(w.B, w.H, w.P, L, w.D).permute(2, 0, 1, 3, 4).contiguous()
    lse = lse.reshape(w.B, w.H, w.P, L).permute(2, 0, 1, 3).contiguous()
    delta = torch.empty_like(lse)
    dq = torch.empty((w.P, w.B, w.H, L, w.D), dtype=torch.float32, device=dev)
    dk = torch.empty((w.P, w.B, w.Hkv, L, w.D), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)

    def step():
        with torch.cuda.stream(stream):
            dq.zero_()
            dk.zero_()
            dv.zero_()
        for rank in range(w.P):
            rm.ring_attn_bwd_delta(o[rank], do[rank], out=delta[rank], stream=stream)
        for t in range(w.P):
            for rank in range(w.P):
                owner = (rank - t) % w.P
                rm.ring_attn_bwd_step(q[rank], k[owner], v[owner], lse[rank], delta[rank],
                                      do[rank], dq[rank], dk[owner], dv[owner], w.P, rank, owner,
                                      w.causal, w.order, stream=stream)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    steps = max(2, min(args.steps, 10))
    ms = time_on_stream(step, steps, stream) / steps
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the backward step benchmark")
    return {"workload": w.name, "ms_per_step": ms, "tflops": w.bwd_flops() / ms / 1e9,
            "launches_per_step": w.P * w.P + w.P + 3, "flops_per_step": w.bwd_flops()}


def bench_exchange(args, dev, stream):
    """The Ulysses exchange-buffer kernels on the 131072-token USP workload's
    shards (U = 4 x R = 4: 16 devices of 8192 tokens): every device's Q, K, V
    packed into its send buffer, and every receive buffer unpacked into the
    device's head shards, 32 launches on this device (the all-to-all between
    them is NCCL's and not part of this)."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS
    w = WORKLOADS["usp_fwd_bf16_S128k_u4r4"]
    U, R = w.ulysses, w.P
    n = U * R
    s = w.S // n
    shards = [[torch.randn((w.B, s, h, w.D), device=dev).to(w.dtype) for h in (w.H, w.Hkv, w.Hkv)]
              for _ in range(n)]
    heads = [w.H, w.Hkv, w.Hkv]
    bufs = [torch.empty((w.H + 2 * w.Hkv) * w.B * s * w.D, device=dev, dtype=w.dtype)
            for _ in range(n)]
    outs = [[torch.empty((w.B, h // U, U * s, w.D), device=dev, dtype=w.dtype) for h in heads]
            for _ in range(n)]

    def step():
        for i in range(n):
            rm.ulysses_pack(shards[i], U, "seq_to_head", buf=bufs[i], stream=stream)
        for i in range(n):
            rm.ulysses_unpack(bufs[i], U, heads, w.B, s, w.D, "seq_to_head", outs=outs[i],
                              stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 50))
    ms = time_on_stream(step, steps, stream) / steps
    moved = 2 * 2 * sum(b.numel() * b.element_size() for b in bufs)  # pack + unpack, read + write
    return {"workload": w.name, "ms_per_step": ms, "bytes_per_step": moved,
            "gbs": moved / ms / 1e6, "launches_per_step": 2 * n}


def bench_masked(args, dev, stream, name):
    """Forward with a sparser mask: the 32k GQA layer with a 4096-key causal
    window, or over packed documents."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS
    w = WORKLOADS[name]
    table = rm.varlen_bounds(list(w.cu_seqlens), w.S, w.causal, device=dev) if w.cu_seqlens \
        else None
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q, k, v = ((torch.randn(s, generator=g, device=dev) * w.input_scale).to(w.dtype)
               for s in [(w.B, w.H, w.S, w.D), (w.B, w.Hkv, w.S, w.D), (w.B, w.Hkv, w.S, w.D)])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)

    def step():
        rm.ring_attn_fwd(q, k, v, w.P, w.causal, w.order, out=o, lse=lse, stream=stream,
                         window=w.window, bounds=table)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 100))
    ms = time_on_stream(step, steps, stream) / steps
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the window benchmark")
    return {"workload": w.name, "window": w.window, "docs": max(len(w.cu_seqlens) - 1, 0),
            "ms_per_launch": ms,
            "tflops": w.fwd_flops() / ms / 1e9, "flops_per_launch": w.fwd_flops(),
            "launches": steps + max(3, args.warmup)}


def bench_backward(args, dev, stream):
    """Ring attention backward on the 64k-token workload (B=2, 16 heads, P=16)."""
    import torch
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200.synth import WORKLOADS
    w = WORKLOADS["ring_fwdbwd_bf16_S64k_causal_zigzag"]
    if args.bwd_heads:
        import dataclasses
        w = dataclasses.replace(w, B=1, H=args.bwd_heads, Hkv=args.bwd_heads,
                                name=f"{w.name}_B1_H{args.bwd_heads}")
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q, k, v, do = ((torch.randn(s, generator=g, device=dev) * w.input_scale).to(w.dtype)
                   for s in [(w.B, w.H, w.S, w.D), (w.B, w.Hkv, w.S, w.D),
                             (w.B, w.Hkv, w.S, w.D), (w.B, w.H, w.S, w.D)])
    o, lse = rm.ring_attn_fwd(q, k, v, w.P, w.causal, w.order, stream=stream)
    ws = torch.empty(rm.native.rm_ring_attn_bwd_workspace_size(w.B, w.H, w.S), dtype=torch.uint8,
                     device=dev)

    def step():
        return rm.ring_attn_bwd(q, k, v, o, lse, do, w.P, w.causal, w.order, workspace=ws,
                                stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
    torch.cuda.synchronize()
    steps = max(2, min(args.steps, 10))
    ms = time_on_stream(step, steps, stream) / steps
    # the fused kernel (dQ by reductions), for comparison
    before = rm.native.rm_get_bwd_deterministic()
    rm.native.rm_set_bwd_deterministic(0)
    try:
        with torch.cuda.stream(stream):
            step()
        torch.cuda.synchronize()
        ms_fused = time_on_stream(step, steps, stream) / steps
    finally:
        rm.native.rm_set_bwd_deterministic(before)
    if rm.native.rm_check_device_status(stream) != 0:
        raise RuntimeError("device watchdog fired during the backward benchmark")
    return {"workload": w.name, "ms_per_step": ms, "tflops": w.bwd_flops() / ms / 1e9,
            "flops_per_step": w.bwd_flops(), "ms_fused": ms_fused,
            "tflops_fused": w.bwd_flops() / ms_fused / 1e9}


def build_line(out, w, args, world, peaks, peak_src):
    """The JSON line (without the CPU baseline) from the measurements in `out`."""
    line = {"metric": METRIC, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) x 0.5, bf16)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup}
    cfg = workload_config(w)
    if "fwd" in out:
        f = out["fwd"]
        ms_step = f["ms_total"] / args.steps
        flops = w.fwd_flops()
        value = world * flops * args.steps / (f["ms_total"] * 1e-3) / 1e12
        sources = ["ring_ulysses_sequence_b200/csrc/fwd_tc.cu",
                   "ring_ulysses_sequence_b200/csrc/common.cuh"]
        peak = peaks["bf16_tflops"]
        achieved = flops / (ms_step * 1e-3) / 1e12
        line.update({
            "value": value, "unit": "TFLOPS", "ms_per_step": ms_step,
            # the denominator is the MEASURED dense bf16 GEMM rate of this pool's
            # B200s (an achieved-GEMM ceiling), not NVIDIA's datasheet figure;
            # both fractions are given
            "pct_of_peak": 100.0 * achieved / peak,
            "pct_of_peak_basis": f"{peak_src} bf16 GEMM ceiling {peak} TFLOPS "
                                 "(torch.matmul 8192^3 burst on this pool's B200s)",
            "pct_of_datasheet_dense_peak": 100.0 * achieved / 2250.0,
            "roofline": {"bound": "tensor", "kernel": "ring_fwd_tc_kernel<128, 0>",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                         "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
                         "frac_of_datasheet_2250": achieved / 2250.0,
                         "flops_per_launch": flops,
                         "traffic": profile_traffic("ring_fwd_tc_S32k_gqa_causal_zigzag.txt",
                                                    sources),
                         "traffic_source": "profiles/ring_fwd_tc_S32k_gqa_causal_zigzag.txt "
                                           "(null when its source digest is not the current "
                                           "sources')"},
            "clocks": f["clocks"],
            "gpu_launches": f["launches"],
        })
        if "e2e" in f:
            e = f["e2e"]
            line["e2e"] = {"value": world * flops / (e["ms_per_step"] * 1e-3) / 1e12,
                           "unit": "TFLOPS", "h2d_bytes_per_step": e["h2d"],
                           "d2h_bytes_per_step": e["d2h"], "ms_per_step": e["ms_per_step"],
                           "steps": e["steps"],
                           "path": "pinned host q,k,v -> H2D -> rm_ring_attn_fwd -> D2H O, LSE; "
                                   "double-buffered on three streams, so step i+1's copy in and "
                                   "step i-1's copy out overlap step i's forward"}
    line["config"] = cfg
    extra = {}
    if "permute" in out:
        p = out["permute"]
        extra["ulysses_permute_qkv"] = {
            "workload": p["workload"], "ms": p["ms_per_launch"], "GB/s": p["gbs"],
            "roofline": {"bound": "hbm", "achieved": p["gbs"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": p["gbs"] / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} hbm_gbs",
                         "bytes_per_launch": p["bytes_per_launch"]}}
    if "layout" in out:
        for name, x in out["layout"].items():
            extra[name] = {
                "workload": f"{w.name} tensors", "ms": x["ms"], "GB/s": x["gbs"],
                "roofline": {"bound": "hbm", "achieved": x["gbs"], "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": x["gbs"] / peaks["hbm_gbs"],
                             "peak_source": f"{peak_src} hbm_gbs",
                             "bytes_per_launch": x["bytes_per_launch"]}}
    if "allgather" in out:
        x = out["allgather"]
        extra["allgather_attn_fwd"] = {
            "workload": x["workload"], "ms_per_step": x["ms_per_step"], "TFLOPS": x["tflops"],
            "ms_attention_only": x["ms_attention"], "TFLOPS_attention_only": x["tflops_attention"],
            "step": "allgather_kv (K, V rank-major -> natural) + rm_allgather_attn_fwd",
            "kv_bytes_resident_per_rank": x["kv_bytes_per_rank"],
            "roofline": {"bound": "tensor", "achieved": x["tflops_attention"],
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": x["tflops_attention"] / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                         "flops_per_launch": x["flops_per_launch"]}}
    if "steps" in out:
        x = out["steps"]
        extra["ring_attn_fwd_step"] = {
            "workload": x["workload"], "ms_per_step": x["ms_per_step"], "TFLOPS": x["tflops"],
            "step": "P ranks x P steps of rm_ring_attn_fwd_step_merge on one device "
                    "(no block exchange)",
            "launches_per_step": x["launches_per_step"],
            "ms_per_step_two_calls": x["ms_per_step_two_calls"],
            "TFLOPS_two_calls": x["tflops_two_calls"],
            "roofline": {"bound": "tensor", "achieved": x["tflops"], "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": x["tflops"] / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                         "flops_per_step": x["flops_per_step"]}}
    if "bwdsteps" in out:
        x = out["bwdsteps"]
        extra["ring_attn_bwd_step"] = {
            "workload": x["workload"], "ms_per_step": x["ms_per_step"], "TFLOPS": x["tflops"],
            "step": "per rank rm_ring_attn_bwd_delta, then P x P rm_ring_attn_bwd_step in the "
                    "reverse ring's schedule on one device (no exchange)",
            "launches_per_step": x["launches_per_step"],
            "roofline": {"bound": "tensor", "achieved": x["tflops"],
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": x["tflops"] / peaks["bf16_tflops_sustained"],
                         "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "flops_per_step": x["flops_per_step"]}}
    if "exchange" in out:
        x = out["exchange"]
        extra["ulysses_pack_unpack"] = {
            "workload": x["workload"], "ms_per_step": x["ms_per_step"], "GB/s": x["gbs"],
            "step": "16 devices' Q/K/V packed into send buffers + 16 receive buffers unpacked "
                    "(rm_ulysses_pack / rm_ulysses_unpack, SEQ_TO_HEAD)",
            "launches_per_step": x["launches_per_step"],
            "roofline": {"bound": "hbm", "achieved": x["gbs"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": x["gbs"] / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} hbm_gbs",
                         "bytes_per_step": x["bytes_per_step"]}}
    for key, label in (("window", "ring_attn_fwd_window"), ("packed", "ring_attn_fwd_varlen")):
        if key not in out:
            continue
        x = out[key]
        extra[label] = {
            "workload": x["workload"], "window": x["window"], "docs": x["docs"],
            "ms": x["ms_per_launch"], "TFLOPS": x["tflops"],
            "roofline": {"bound": "tensor", "achieved": x["tflops"], "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": x["tflops"] / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                         "flops_per_launch": x["flops_per_launch"],
                         "flops_rule": "4 B H D x visible (query, key) pairs"}}
    if "bwd" in out:
        b = out["bwd"]
        if "unavailable" in b:
            extra["ring_attn_bwd"] = b
        else:
            extra["ring_attn_bwd"] = {
                "workload": b["workload"], "ms": b["ms_per_step"], "TFLOPS": b["tflops"],
                "kernels": "two kernels, every element written once (rm_set_bwd_deterministic(1), "
                           "the default)",
                "ms_fused": b.get("ms_fused"), "TFLOPS_fused": b.get("tflops_fused"),
                "kernels_fused": "one kernel, dQ added by TMA reductions in a run-dependent "
                                 "order (rm_set_bwd_deterministic(0))",
                "roofline": {"bound": "tensor", "achieved": b["tflops"],
                             "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                             "frac": b["tflops"] / peaks["bf16_tflops_sustained"],
                             "frac_fused": (b["tflops_fused"] / peaks["bf16_tflops_sustained"]
                                            if b.get("tflops_fused") else None),
                             "peak_source": f"{peak_src} bf16_tflops_sustained"}}
    if extra:
        line["extra"] = extra
    return line


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    from ring_ulysses_sequence_b200 import multi
    from ring_ulysses_sequence_b200.synth import BENCH_WORKLOAD, WORKLOADS
    rank, world, local = multi.env_ranks()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    multi.init("nccl", timeout_s=120, device=dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    w = WORKLOADS[BENCH_WORKLOAD]
    out = {}
    try:
        if args.only in ("all", "fwd"):
            out["fwd"] = bench_forward(w, args, dev, stream)
        if rank == 0 and args.only in ("all", "permute"):
            out["permute"] = bench_permute(args, dev, stream)
        if rank == 0 and args.only in ("all", "layout"):
            out["layout"] = bench_layout(args, dev, stream)
        if rank == 0 and args.only in ("all", "allgather"):
            out["allgather"] = bench_allgather(args, dev, stream)
        if rank == 0 and args.only in ("all", "steps"):
            out["steps"] = bench_steps(args, dev, stream)
        if rank == 0 and args.only in ("all", "bwdsteps"):
            out["bwdsteps"] = bench_bwd_steps(args, dev, stream)
        if rank == 0 and args.only in ("all", "exchange"):
            out["exchange"] = bench_exchange(args, dev, stream)
        if rank == 0 and args.only in ("all", "window"):
            out["window"] = bench_masked(args, dev, stream,
                                         "ring_fwd_bf16_S32k_gqa_causal_zigzag_window4k")
        if rank == 0 and args.only in ("all", "packed"):
            out["packed"] = bench_masked(args, dev, stream,
                                         "ring_fwd_bf16_S32k_gqa_causal_zigzag_packed")
        if rank == 0 and args.only in ("all", "bwd"):
            try:
                out["bwd"] = bench_backward(args, dev, stream)
            except Exception as e:  # backward not available: say so in the line
                out["bwd"] = {"unavailable": str(e)[:200]}
    finally:
        multi.barrier(dev)
    if rank != 0:
        multi.shutdown()
        return

    line = build_line(out, w, args, world, peaks, peak_src)
    if world == 1 and not args.skip_cpu and args.only in ("all", "fwd"):
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    multi.shutdown()


if __name__ == "__main__":
    main()
