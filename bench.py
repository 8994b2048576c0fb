#!/usr/bin/env python
"""Benchmark of the exact tiled attention hot path on B200.

One step is the whole path on one batch of the causal GQA prefill workload
(B=2, N=8192, Hq=32, Hkv=8, d=128, bf16, causal): fa_fwd (O and L), then
fa_bwd (D = rowsum(dO o O), the recompute kernel, dQ convert). Inputs are
seeded synthetic N(0,1) tensors, resident in device memory before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0). FLOPs follow the FlashAttention convention:
fwd = 4 Nq Nk d per (batch, query head), halved for causal; bwd = 2.5 fwd.
With N > 1 (torchrun, one rank per GPU) every rank runs its own independent
batch (the path has no exchange step: replicas, weak scaling); the time is the
max over ranks.

--impl reference times the fp64 CPU oracle (the plain definition) on a
bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(name="causal_gqa_prefill_fwd_bwd", B=2, N=8192, Hq=32, Hkv=8, d=128, dtype="bf16", causal=True)
METRIC = "attention fwd+bwd TFLOPS on 1 B200 (FlashAttention FLOP convention) and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# CPU sample for the oracle: batch 0, every query head, the first T tokens.
# Under the causal mask these tokens form exactly the top-left block of the
# full problem, i.e. a causal attention problem of length T. The CPU-baseline
# leg of the GPU run takes one larger sample; the reference arm repeats a
# smaller one per step so that a whole --steps/--warmup run stays short.
CPU_SAMPLE_TOKENS = 2048
REF_STEP_TOKENS = 1024
# Small case of the same kernels for profiler captures (inputs still > L2).
PROFILE_CASE = dict(B=1, N=4096)


def flops_fwd(B, N, Hq, d, causal):
    f = 4.0 * N * N * d * B * Hq
    return f / 2 if causal else f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def choose_peak(clocks, peaks, peak_src):
    """The bf16 peak that matches the timed region's clocks: the burst figure (measured
    with the GPU at its maximum SM clock) when the region's median SM clock under load
    is within 5 % of the maximum or no clock record exists; the sustained figure
    (measured over seconds at the 1 kW power cap) when the clocks sat lower."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if clocks and clocks.get("sm_max_mhz") and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"]:
        return sust, (f"bf16_tflops_sustained ({peak_src}): median SM clock {clocks['sm_mhz']:.0f} MHz under "
                      f"load, below the {clocks['sm_max_mhz']:.0f} MHz maximum")
    why = (f"median SM clock {clocks['sm_mhz']:.0f} of {clocks['sm_max_mhz']:.0f} MHz under load" if clocks
           else "no clock record")
    return burst, f"bf16_tflops burst ({peak_src}): {why}"


def algorithmic_bytes(kernel, B, N, Hq, Hkv, d):
    """Bytes a launch must move at least: the backward main kernel reads Q, dO, K, V, L
    and D and writes dK and dV (the fp32 dQ accumulator's reductions are implementation
    traffic, not counted); the forward reads Q, K, V and writes O and L."""
    q_b, kv_b, row_b = 2 * B * N * Hq * d, 2 * B * N * Hkv * d, 4 * B * Hq * N
    if kernel == "fa_bwd128_kernel":
        return 2 * q_b + 4 * kv_b + 2 * row_b
    return 2 * q_b + 2 * kv_b + row_b


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_tiny_single_core():
    """The oracle's forward of the tiny workload (B=1, H=2, N=256, d=64) on one core."""
    import oracle
    from exact_tiled_attention_36_b200 import inputs
    cfg = inputs.TINY
    fi = inputs.make_fixed(cfg)
    args = [oracle._f64(t) for t in (fi.q, fi.k, fi.v)]
    before = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        oracle.attn_fwd(*args, cfg.scale, cfg.causal)
        t0 = time.perf_counter()
        oracle.attn_fwd(*args, cfg.scale, cfg.causal)
        dt = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(before)
    flops = flops_fwd(cfg.B, cfg.Nq, cfg.Hq, cfg.d, cfg.causal)
    return {"seconds": dt, "tflops": flops / dt / 1e12, "cores": 1,
            "sample": "oracle forward of the whole tiny workload"}


# The device code each profiled kernel is compiled from (its header and what it
# includes; the host file only encodes descriptors and launches).
KERNEL_SOURCES = {
    "fa_fwd_kernel": ("sm100.cuh", "fa_fwd.cuh"),
    "fa_bwd128_kernel": ("sm100.cuh", "fa_bwd.cuh", "fa_bwd128.cuh"),
    "fa_decode_narrow_kernel": ("sm100.cuh", "fa_decode.cuh"),
}


def csrc_digest(kernel=None):
    """sha256 (16 hex digits) of `kernel`'s source files (every csrc file if None)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "exact_tiled_attention_36_b200", "csrc")
    names = sorted(os.listdir(d)) if kernel is None else sorted(KERNEL_SOURCES[kernel])
    for name in names:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was
    captured from the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}.txt")
    try:
        kv = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("csrc_sha256_16") == csrc_digest(kernel):
            return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load)}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def any_rank_throttled(clocks, world, device):
    """Whether any rank's clock record (ClockSampler.stop()) shows a throttle reason
    that rejects the measurement. Every rank gets the same answer, so all of them
    re-measure together and take the same collective steps (one all-reduce per call
    on every rank when world > 1)."""
    bad = 1.0 if clocks and (set(clocks["reasons"]) & BAD_REASONS) else 0.0
    return max_over_ranks(bad, world, device) > 0.0


# ----------------------------------------------------------------------------- multi-rank plumbing
def rank_seed(base_seed, rank):
    """Each rank draws its own batch: independent replicas of the workload."""
    return base_seed + 1000 * rank


def max_over_ranks(x, world, device):
    """The largest of every rank's `x` (the job's time is its slowest rank's)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, flops_per_step, steps, max_ms):
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_step * steps / (max_ms / 1e3) / 1e12


# ----------------------------------------------------------------------------- CPU oracle (reference arm)
def cpu_oracle_sample(n_steps, tokens):
    """Time the fp64 oracle (fwd + bwd) on the bounded sample, n_steps times."""
    import oracle
    from exact_tiled_attention_36_b200 import inputs
    w = WORKLOAD
    cfg = inputs.CAUSAL_GQA
    fi = inputs.make_fixed(cfg, B=1, Nq=tokens, Nk=tokens)
    args = [oracle._f64(t) for t in (fi.q, fi.k, fi.v, fi.do)]
    oracle.build()
    flops = 3.5 * flops_fwd(1, tokens, w["Hq"], w["d"], w["causal"])
    times = []
    for _ in range(n_steps):
        t0 = time.perf_counter()
        oracle.attn_fwd(args[0], args[1], args[2], cfg.scale, True)
        oracle.attn_bwd(args[0], args[1], args[2], args[3], cfg.scale, True)
        times.append(time.perf_counter() - t0)
    return flops, times, oracle.num_threads()


def cpu_sample_desc(tokens):
    w = WORKLOAD
    return (f"oracle fwd+bwd (fp64, OpenMP) on batch 0, all {w['Hq']} query heads / {w['Hkv']} KV heads, "
            f"first {tokens} of {w['N']} tokens (the top-left causal block), d={w['d']}")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.warmup > 0:
        cpu_oracle_sample(args.warmup, REF_STEP_TOKENS)
    flops, times, cores = cpu_oracle_sample(args.steps, REF_STEP_TOKENS)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "sample_tokens": REF_STEP_TOKENS,
                   **{k: WORKLOAD[k] for k in ("Hq", "Hkv", "d", "causal")}},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": cpu_sample_desc(REF_STEP_TOKENS) + ", once per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    from exact_tiled_attention_36_b200 import binding as fb
    from exact_tiled_attention_36_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()


    fb.lib()
    w = dict(WORKLOAD)
    if args.profile_small:
        w.update(PROFILE_CASE)
    cfg = inputs.CAUSAL_GQA
    # each rank draws its own batch (independent replicas of the workload)
    fi = inputs.make_fixed(cfg, seed=rank_seed(cfg.seed, rank), B=w["B"], Nq=w["N"], Nk=w["N"])
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    scale = d ** -0.5
    dt = fb.FA_BF16
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def step():
        st = fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                       scale, 1, dt, sh)
        if st != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(st))
        st = fb.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                       dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, N, d, scale, 1, dt,
                       sh)
        if st != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(st))

    f_fwd = flops_fwd(B, N, Hq, d, True)
    f_step = 3.5 * f_fwd
    warm = max(args.warmup, 3)
    K = args.steps

    def timed_region():
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
        for e in ev:
            for x in e:
                x.record(stream)  # create the underlying events
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(K):
            e0, e1, e2, eb0, eb1 = ev[i]
            fb.fa_bwd_set_timing_events(eb0.cuda_event, eb1.cuda_event)
            e0.record(stream)
            st = fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N,
                           d, scale, 1, dt, sh)
            e1.record(stream)
            st2 = fb.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, N, d, scale,
                            1, dt, sh)
            e2.record(stream)
            if st != fb.FA_OK or st2 != fb.FA_OK:
                raise RuntimeError(fb.fa_status_string(st or st2))
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        fb.fa_bwd_set_timing_events(None, None)
        total_ms = start.elapsed_time(end)
        fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
        bwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
        bwd_main_ms = [e[3].elapsed_time(e[4]) for e in ev]
        return total_ms, fwd_ms, bwd_ms, bwd_main_ms

    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    if fb.fa_get_last_device_error(None) != fb.FA_OK:
        raise RuntimeError("device error during warm-up")
    if args.profile_small:  # profiler driver: the warm-up launches are the capture targets
        print(f"profile case B={B} N={N}: {warm} fwd+bwd steps done", flush=True)
        return 0

    sampler = ClockSampler(local)
    result = None
    clocks = None
    for attempt in range(2):
        sampler.start()
        time.sleep(0.3)
        result = timed_region()
        clocks = sampler.stop()
        if not any_rank_throttled(clocks, world, "cuda"):
            break
    total_ms, fwd_ms, bwd_ms, bwd_main_ms = result
    if fb.fa_get_last_device_error(None) != fb.FA_OK:
        raise RuntimeError("device error during the timed region")
    total_ms = max_over_ranks(total_ms, world, "cuda")

    # The forward's own metric: forward calls back to back (no backward between them, so
    # the GPU is not held at the power cap the step loop settles at); the tensors touched
    # per call (~340 MB) are larger than the L2.
    n_fwd = max(10, min(3 * K, 30))

    def fwd_call():
        st = fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                       scale, 1, dt, sh)
        if st != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(st))

    torch.cuda.synchronize()
    time.sleep(0.5)  # let the clocks recover from the step loop
    for _ in range(3):
        fwd_call()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(n_fwd):
        fwd_call()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    fwd_alone_ms = max_over_ranks(f0.elapsed_time(f1), world, "cuda") / n_fwd

    # End to end through the C ABI with host buffers: every step copies its q, k, v, dO
    # in from pinned host memory and its dq, dk, dv out, as a training input pipeline
    # would: three streams and two buffer slots, so that the copies of step i + 1 (in)
    # and step i - 1 (out) cross PCIe while step i's kernels run.
    hq, hk, hv, hdo = (t.pin_memory() for t in (fi.q, fi.k, fi.v, fi.do))
    h_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (q, k, v)] for _ in range(2)]
    d_in = [[q, k, v, do], [torch.empty_like(t) for t in (q, k, v, do)]]
    d_out = [[dq, dk, dv], [torch.empty_like(t) for t in (dq, dk, dv)]]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in h_out[0])
    K_e2e = max(3, min(K, 20))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_run, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    used = [False, False]

    def run_slot(b):
        qq, kk, vv, dd = (t.data_ptr() for t in d_in[b])
        gq, gk, gv = (t.data_ptr() for t in d_out[b])
        st = fb.fa_fwd(qq, kk, vv, o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d, scale, 1, dt, sh)
        st2 = fb.fa_bwd(qq, kk, vv, o.data_ptr(), lse.data_ptr(), dd, gq, gk, gv, ws.data_ptr(), B, Hq, Hkv, N, N,
                        d, scale, 1, dt, sh)
        if st != fb.FA_OK or st2 != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(st or st2))

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            if used[b]:
                s_in.wait_event(ev_run[b])  # step i - 2 has read this slot's inputs
            with torch.cuda.stream(s_in):
                for dst, src in zip(d_in[b], (hq, hk, hv, hdo)):
                    dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if used[b]:
                stream.wait_event(ev_out[b])  # step i - 2's gradients have left this slot
            run_slot(b)
            ev_run[b].record(stream)
            s_out.wait_event(ev_run[b])
            with torch.cuda.stream(s_out):
                for dst, src in zip(h_out[b], d_out[b]):
                    dst.copy_(src, non_blocking=True)
            ev_out[b].record(s_out)
            used[b] = True

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(s_in)  # every copy and kernel below is ordered after it through the events
    e2e_steps(K_e2e)
    s1.record(s_out)  # the last read-back waits for the last step, which waited for its inputs
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(s0.elapsed_time(s1), world, "cuda")

    peaks, peak_src = load_peaks()
    value = job_tflops(world, f_step, K, total_ms)
    e2e_value = job_tflops(world, f_step, K_e2e, e2e_ms)
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms)
    main_avg = statistics.mean(bwd_main_ms)
    f_bwd = 2.5 * f_fwd
    # dominant kernel: the longer of the forward kernel and the backward main kernel
    if main_avg >= fwd_avg:  # d = 128: the backward main kernel
        kname, kflops, kms = "fa_bwd128_kernel", f_bwd, main_avg
    else:
        kname, kflops, kms = "fa_fwd_kernel", f_fwd, fwd_avg
    achieved = kflops / (kms / 1e3) / 1e12
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak, peak_kind = choose_peak(clocks, peaks, peak_src)
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    clock_mhz = clocks["sm_mhz"] if clocks else peaks.get("sm_max_mhz", 1965.0)
    f_tf, b_tf = f_fwd / (fwd_avg / 1e3) / 1e12, f_bwd / (bwd_avg / 1e3) / 1e12
    traffic = profiled_traffic(kname)
    alg_bytes = algorithmic_bytes(kname, B, N, Hq, Hkv, d)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": warm,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w["name"], "B": B, "seq_len": N, "Hq": Hq, "Hkv": Hkv, "d": d, "causal": True,
                   "parallelism": f"replicas x{world} (no exchange step)",
                   "l2": "inputs larger than L2: ~1.0 GB of tensors touched per step vs 126 MB L2"},
        "fwd_tflops": f_tf, "bwd_tflops": b_tf,
        # the fraction of the peak the clock record selects (roofline.peak_kind), and of both
        "fwd_frac": f_tf / peak, "bwd_frac": b_tf / peak,
        "fwd_frac_of_burst": f_tf / peak_burst, "bwd_frac_of_burst": b_tf / peak_burst,
        "fwd_frac_of_sustained": f_tf / peak_sust, "bwd_frac_of_sustained": b_tf / peak_sust,
        "fwd_ms": fwd_avg, "bwd_ms": bwd_avg, "bwd_main_kernel_ms": main_avg,
        "fwd_alone": {"calls": n_fwd, "ms": fwd_alone_ms, "tflops": f_fwd / (fwd_alone_ms / 1e3) / 1e12,
                      "frac_of_burst": f_fwd / (fwd_alone_ms / 1e3) / 1e12 / peak_burst,
                      "how": "forward calls back to back after the step loop, CUDA events, max over ranks"},
        "roofline": {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "peak_burst": peak_burst, "frac_of_burst": achieved / peak_burst,
                     "peak_sustained": peak_sust, "frac_of_sustained": achieved / peak_sust,
                     "traffic": traffic, "algorithmic_bytes": alg_bytes,
                     "traffic_over_algorithmic": (traffic / alg_bytes) if traffic else None},
        "ceilings": {
            "how": "MUFU ex2: 16 per clock per SM x SMs x median SM clock of the timed region x FLOPs per "
                   "score (one exponential per score; 4d FLOP forward, 10d backward)",
            "sms": sms, "sm_mhz": clock_mhz,
            "mufu_fwd_d128_tflops": mufu_ceiling_tflops(128, 4 * 128, sms, clock_mhz),
            "mufu_fwd_d64_tflops": mufu_ceiling_tflops(64, 4 * 64, sms, clock_mhz),
            "mufu_bwd_d128_tflops": mufu_ceiling_tflops(128, 10 * 128, sms, clock_mhz),
            "fwd_frac_of_mufu": f_tf / mufu_ceiling_tflops(d, 4 * d, sms, clock_mhz),
            "bwd_main_frac_of_mufu": (f_bwd / (main_avg / 1e3) / 1e12) / mufu_ceiling_tflops(d, 10 * d, sms,
                                                                                              clock_mhz),
        },
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": K_e2e, "ms_per_step": e2e_ms / K_e2e,
                "how": "pinned host buffers; H2D of q, k, v, dO and D2H of dq, dk, dv every step on their own "
                       "streams, overlapping the neighbouring steps' kernels (two buffer slots)"},
        "gpu_launches": K * 4,  # per step: forward, preprocess, main backward, dQ convert
        "clocks": clocks,
    }
    if world == 1 and not args.no_configs:
        # Every workload and pass, timed after the step loop (CUDA events, inputs resident
        # in device memory): the short-sequence shapes, varlen, the prefill variants, FP8,
        # windows and decode.
        del q, k, v, do, o, lse, dq, dk, dv, ws, d_in, d_out, h_out, hq, hk, hv, hdo
        torch.cuda.empty_cache()
        configs = {}
        Sweep(fb, torch, peaks, configs.__setitem__, sms, clock_mhz).run()
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, times, cores = cpu_oracle_sample(1, CPU_SAMPLE_TOKENS)
        cpu_v = flops / times[0] / 1e12
        line["cpu_baseline"] = {"value": cpu_v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "cpu_model": cpu_model(), "sample": cpu_sample_desc(CPU_SAMPLE_TOKENS),
                                "seconds": times[0], "single_core_tiny": cpu_tiny_single_core()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- per-workload sweep
EX2_PER_CLK_PER_SM = 16  # MUFU exponentials per clock per SM


def mufu_ceiling_tflops(d, flops_per_score, sms, clock_mhz):
    """The TFLOP/s at which the exponentials alone (one per score: the softmax of
    "FlashAttention/zh", section "FlashAttention algorithm") would fill the MUFU pipe:
    16 ex2 / clock / SM x SMs x clock x the FLOPs a score carries (4d forward, 10d
    backward)."""
    return EX2_PER_CLK_PER_SM * sms * clock_mhz * 1e6 * flops_per_score / 1e12


class Sweep:
    """Times the forward (and backward where the workload has one) of every workload
    and the decode workloads. Each result goes to `sink(key, entry)`."""

    def __init__(self, fb, torch, peaks, sink, sms, clock_mhz, only=None):
        self.fb, self.torch, self.sink, self.only = fb, torch, sink, only
        self.peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        self.hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        self.sms, self.clock = sms, clock_mhz
        self.stream = torch.cuda.current_stream()

    def time_it(self, fn, iters):
        torch, fb = self.torch, self.fb
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(iters):
            fn()
        e1.record(self.stream)
        torch.cuda.synchronize()
        if fb.fa_get_last_device_error(None) != fb.FA_OK:
            raise RuntimeError("device error")
        return e0.elapsed_time(e1) / iters

    def emit(self, name, what, ms, flops, nbytes, d=None, fp8=False):
        tf = flops / (ms / 1e3) / 1e12
        e = {"workload": name, "pass": what, "ms": ms, "tflops": tf, "frac_of_burst": tf / self.peak,
             "algorithmic_gbs": nbytes / (ms / 1e3) / 1e9, "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / self.hbm}
        if d is not None:
            per_score = (10 if what == "bwd" else 4) * d
            ceil = mufu_ceiling_tflops(d, per_score, self.sms, self.clock)
            e["mufu_ceiling_tflops"] = ceil
            e["frac_of_mufu_ceiling"] = tf / ceil
        if fp8:  # the E4M3 tensor peak: the measured bf16 burst peak x the nominal 2x ratio
            e["frac_of_fp8_peak"] = tf / (2.0 * self.peak)
        self.sink(f"{name}:{what}", e)

    def want(self, name):
        return self.only is None or self.only in name

    def run(self):
        from exact_tiled_attention_36_b200 import inputs
        fb, torch = self.fb, self.torch
        for cfg in (inputs.TINY, inputs.VISION, inputs.VIT_RMSNORM, inputs.CAUSAL_GQA):
            if not self.want(cfg.name):
                continue
            fi = inputs.make_fixed(cfg)
            q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
            B, N, Hq, d = q.shape
            o, lse = fb.attention_fwd(q, k, v, cfg.scale, cfg.causal)
            flops = flops_fwd(B, N, Hq, d, cfg.causal)
            nbytes = 2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel()
            iters = 1000 if cfg is inputs.TINY else 30
            ms = self.time_it(lambda: fb.attention_fwd(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse), iters)
            self.emit(cfg.name, "fwd", ms, flops, nbytes, d)
            if cfg is inputs.TINY:
                self.tiny_calls(fb, torch, cfg, q, k, v, o, lse, flops, nbytes, d)
            if cfg.backward:
                do = fi.do.cuda()
                ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")
                ms = self.time_it(lambda: fb.attention_bwd(q, k, v, o, lse, do, cfg.scale, cfg.causal, workspace=ws),
                                  20)
                self.emit(cfg.name, "bwd", ms, 2.5 * flops,
                          nbytes + 2 * (do.numel() + q.numel() + k.numel() + v.numel()), d)
            del q, k, v, o, lse, fi
        args = (inputs, fb, torch, self.stream, self.time_it, self.emit)
        if self.want(inputs.CAUSAL_GQA_FP8.name):
            sweep_fp8(inputs.CAUSAL_GQA_FP8, *args)
        if self.want(inputs.CAUSAL_GQA.name + "_window1024_anchor4"):
            sweep_window(*args)
        if self.want("causal_gqa_b2_n8192_hq32_hkv8_d128_noncausal") or \
                self.want("causal_gqa_b2_n8192_hq32_hkv32_d128_mha"):
            sweep_prefill_variants(*args)
        if self.want(inputs.VIT_RMSNORM.name + "_packed_qkv_fused_qk_rmsnorm"):
            sweep_vit_variants(*args)
        for cfg in (inputs.VARLEN, inputs.VARLEN_KEYPAD):
            if self.want(cfg.name):
                sweep_varlen(cfg, *args)
        for cfg, page in ((inputs.DECODE, 0), (inputs.DECODE_RAGGED, 0), (inputs.DECODE_RAGGED, 64),
                          (inputs.DECODE_RAGGED, 32), (inputs.DECODE_RAGGED, 16), (inputs.DECODE_D64, 0),
                          (inputs.DECODE_SPEC4, 0)):
            if self.want(cfg.name + (f"_paged{page}" if page else "")):
                sweep_decode(cfg, page, *args)

    def tiny_calls(self, fb, torch, cfg, q, k, v, o, lse, flops, nbytes, d):
        """The tiny workload is bound by per-call host work when called eagerly: timed
        through the torch-level binding, through the C ABI directly (arguments marshalled
        once), and replayed from a CUDA graph of 100 calls (the device's time per call)."""
        B, N, Hq, _ = q.shape
        Hkv = k.shape[2]
        sh = self.stream.cuda_stream
        f = fb.lib().fa_fwd
        argv = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                float(cfg.scale), int(cfg.causal), fb.FA_BF16, sh)
        if f(*argv) != fb.FA_OK:
            raise RuntimeError("fa_fwd failed")
        ms = self.time_it(lambda: f(*argv), 1000)
        self.emit(cfg.name, "fwd_eager_c_abi", ms, flops, nbytes, d)
        g = torch.cuda.CUDAGraph()
        gs = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=gs):
            for _ in range(100):
                fb.attention_fwd(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse, stream=gs)
        ms = self.time_it(g.replay, 10) / 100
        self.emit(cfg.name, "fwd_graph_replay", ms, flops, nbytes, d)
        del g


# Workloads whose forward kernel gets its own profiler capture: (input config name, calls).
# name -> (workload, calls, overrides of its shape); cases ending in "_bwd_small" run the
# backward after each forward
PROFILE_CASES = {"vision_fwd": ("VISION", 3, {}), "vit_fwd": ("VIT_RMSNORM", 3, {}), "tiny_fwd": ("TINY", 3, {}),
                 "mha_bwd_small": ("CAUSAL_GQA", 3, dict(B=1, Nq=4096, Nk=4096, Hkv=32))}


def run_profile_case(name):
    """A few forward calls of one workload at full size (each holds ~211 MB on the
    device), for ncu captures of the forward kernel on that shape; or, for a backward
    case, a few forward + backward calls of a small prefill shape (~0.3 GB)."""
    import torch
    from exact_tiled_attention_36_b200 import binding as fb
    from exact_tiled_attention_36_b200 import inputs
    cfg_name, calls, over = PROFILE_CASES[name]
    cfg = getattr(inputs, cfg_name)
    backward = name.endswith("_bwd_small")
    fi = inputs.make_fixed(cfg, with_do=backward, **over)
    q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
    do = fi.do.cuda() if backward else None
    o, lse = fb.attention_fwd(q, k, v, cfg.scale, cfg.causal)
    ws = None
    for i in range(calls):
        if i:
            fb.attention_fwd(q, k, v, cfg.scale, cfg.causal, out=o, lse=lse)
        if backward:
            if ws is None:
                ws = torch.empty(fb.fa_bwd_workspace_size(q.shape[0], q.shape[2], q.shape[1], q.shape[3]),
                                 dtype=torch.uint8, device="cuda")
            fb.attention_bwd(q, k, v, o, lse, do, cfg.scale, cfg.causal, workspace=ws)
    torch.cuda.synchronize()
    if fb.fa_get_last_device_error(None) != fb.FA_OK:
        raise RuntimeError("device error")
    what = "forward + backward" if backward else "forward"
    print(f"profile case {name} ({cfg.name}, {over or 'full size'}): {calls} {what} calls done", flush=True)
    return 0


def run_sweep(args):
    """--all-configs: one JSON line per workload and pass (the same entries the default
    bench line carries in its `configs` object)."""
    import torch
    from exact_tiled_attention_36_b200 import binding as fb
    peaks, peak_src = load_peaks()
    fb.lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    clock = peaks.get("sm_max_mhz", 1965.0)

    def sink(key, e):
        print(json.dumps({"kind": "config_sweep", **e, "peaks": peak_src}), flush=True)

    Sweep(fb, torch, peaks, sink, sms, clock, args.only).run()
    return 0


def sweep_fp8(cfg, inputs, fb, torch, stream, time_it, emit):
    f8 = inputs.make_fp8(cfg)
    q8, k8, v8 = f8.q.cuda(), f8.k.cuda(), f8.v.cuda()
    qs, ks, vs = f8.q_scale.cuda(), f8.k_scale.cuda(), f8.v_scale.cuda()
    B, N, Hq, d = q8.shape
    Hkv = k8.shape[2]
    o = torch.empty((B, N, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")

    def ffp8():
        r = fb.fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), qs.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                          o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d, cfg.scale, int(cfg.causal),
                          stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    emit(cfg.name, "fwd", time_it(ffp8, 30), flops_fwd(B, N, Hq, d, cfg.causal),
         q8.numel() + k8.numel() + v8.numel() + 2 * o.numel() + 4 * lse.numel(), d, fp8=True)


def sweep_window(inputs, fb, torch, stream, time_it, emit):
    """Local attention: the causal GQA prefill shape with a causal sliding window of 1024
    keys, alone and with 4 global anchor keys."""
    cfg = inputs.CAUSAL_GQA
    fi = inputs.make_fixed(cfg)
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    wl, wr = 1024, 0
    pairs = sum(min(i + 1, wl + 1) for i in range(N))  # visible (query, key) pairs per (batch, head)
    wflops = 4.0 * d * pairs * B * Hq
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")

    def wfwd():
        r = fb.fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N,
                             N, d, cfg.scale, wl, wr, fb.FA_BF16, stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    def wbwd():
        r = fb.fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, N, d,
                             cfg.scale, wl, wr, fb.FA_BF16, stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    nb = 2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel()
    emit(cfg.name + "_window1024", "fwd", time_it(wfwd, 30), wflops, nb, d)
    emit(cfg.name + "_window1024", "bwd", time_it(wbwd, 20), 2.5 * wflops,
         nb + 2 * (do.numel() + q.numel() + k.numel() + v.numel()), d)
    # the same window plus 4 global anchor keys (the first tokens, visible to every query)
    na = 4
    apairs = pairs + sum(max(0, min(na, i - wl)) for i in range(N))
    aflops = 4.0 * d * apairs * B * Hq

    def afwd():
        r = fb.fa_fwd_window_anchor(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
                                    Hkv, N, N, d, cfg.scale, wl, wr, na, fb.FA_BF16, stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    def abwd():
        r = fb.fa_bwd_window_anchor(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq,
                                    Hkv, N, N, d, cfg.scale, wl, wr, na, fb.FA_BF16, stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    emit(cfg.name + "_window1024_anchor4", "fwd", time_it(afwd, 30), aflops, nb, d)
    emit(cfg.name + "_window1024_anchor4", "bwd", time_it(abwd, 20), 2.5 * aflops,
         nb + 2 * (do.numel() + q.numel() + k.numel() + v.numel()), d)


def sweep_prefill_variants(inputs, fb, torch, stream, time_it, emit):
    """The causal GQA prefill shape without the causal mask, and with as many KV heads
    as query heads (Hq = Hkv = 32): the d = 128 figures beside the causal GQA ones."""
    base = inputs.CAUSAL_GQA
    for tag, causal, hkv in (("_noncausal", False, base.Hkv), ("_mha", True, base.Hq)):
        fi = inputs.make_fixed(base, causal=causal, Hkv=hkv)
        q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
        B, N, Hq, d = q.shape
        flops = flops_fwd(B, N, Hq, d, causal)
        o, lse = fb.attention_fwd(q, k, v, base.scale, causal)
        ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")
        nb = 2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel()
        emit(base.name.replace("_hkv8", f"_hkv{hkv}") + tag, "fwd",
             time_it(lambda: fb.attention_fwd(q, k, v, base.scale, causal, out=o, lse=lse), 30), flops, nb, d)
        emit(base.name.replace("_hkv8", f"_hkv{hkv}") + tag, "bwd",
             time_it(lambda: fb.attention_bwd(q, k, v, o, lse, do, base.scale, causal, workspace=ws), 20),
             2.5 * flops, nb + 2 * (do.numel() + q.numel() + k.numel() + v.numel()), d)
        del q, k, v, do, o, lse, ws, fi


def sweep_vit_variants(inputs, fb, torch, stream, time_it, emit):
    """The ViT workload through the packed-QKV layout (B, S, 3, H, d), O written as
    (B, H, S, d); and from raw Q and K with their RMS normalisation fused."""
    cfg = inputs.VIT_RMSNORM
    fi = inputs.make_fixed(cfg)
    qkv = torch.stack([fi.q, fi.k, fi.v], dim=2).cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    B, N, Hq, d = q.shape
    o = torch.empty((B, Hq, N, d), dtype=q.dtype, device="cuda").permute(0, 2, 1, 3)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    st3 = lambda t: tuple(t.stride()[:3])

    def packed():
        r = fb.fa_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), st3(q),
                              st3(k), st3(v), st3(o), B, Hq, Hq, N, N, d, cfg.scale, int(cfg.causal), fb.FA_BF16,
                              stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    ms = time_it(packed, 30)
    emit(cfg.name + "_packed_qkv", "fwd", ms, flops_fwd(B, N, Hq, d, cfg.causal),
         2 * (q.numel() + k.numel() + v.numel() + q.numel()) + 4 * lse.numel(), d)
    del qkv, q, k, v, o, lse
    # the ViT workload with raw Q and K, their RMS normalisation fused (fa_fwd_qk_rmsnorm)
    cfg = inputs.VIT_RMSNORM
    fi = inputs.make_fixed(cfg, rmsnorm=False)
    q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
    B, N, Hq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    ws = torch.empty(fb.fa_fwd_qk_rmsnorm_workspace_size(B, N, Hq, d), dtype=torch.uint8, device="cuda")

    def fused():
        r = fb.fa_fwd_qk_rmsnorm(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 ws.data_ptr(), B, Hq, Hq, N, N, d, cfg.scale, int(cfg.causal), inputs.RMSNORM_EPS,
                                 fb.FA_BF16, stream.cuda_stream)
        if r != fb.FA_OK:
            raise RuntimeError(fb.fa_status_string(r))

    ms = time_it(fused, 30)
    emit(cfg.name + "_fused_qk_rmsnorm", "fwd", ms, flops_fwd(B, N, Hq, d, cfg.causal),
         2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel(), d)



def sweep_varlen(cfg, inputs, fb, torch, stream, time_it, emit):
    vi = inputs.make_varlen(cfg)
    q, k, v = (t.cuda() for t in (vi.q, vi.k, vi.v))
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    o, lse = fb.attention_varlen_fwd(q, k, v, cu_q, cu_k, vi.max_seqlen_q, vi.max_seqlen_k, cfg.scale, cfg.causal)
    flops = sum(4.0 * lq * lk * cfg.d * cfg.Hq for lq, lk in zip(vi.seqlens_q, vi.seqlens_k))
    nbytes = 2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel()
    ms = time_it(lambda: fb.attention_varlen_fwd(q, k, v, cu_q, cu_k, vi.max_seqlen_q, vi.max_seqlen_k,
                                                 cfg.scale, cfg.causal, out=o, lse=lse), 20)
    emit(cfg.name, "fwd", ms, flops, nbytes, cfg.d)
    if cfg is inputs.VARLEN:
        # the varlen backward on the same packed batch (dO drawn after Q, K, V)
        do = inputs.make_varlen(cfg, with_do=True).do.cuda()
        n, Tq, Tk = len(vi.seqlens_q), q.shape[0], k.shape[0]
        ws = torch.empty(fb.fa_varlen_bwd_workspace_size(n, Tq, vi.max_seqlen_q, cfg.Hq, cfg.d),
                         dtype=torch.uint8, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16

        def vbwd():
            st = fb.fa_varlen_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                                  cu_q.data_ptr(), cu_k.data_ptr(), n, Tq, Tk, vi.max_seqlen_q,
                                  vi.max_seqlen_k, cfg.Hq, cfg.Hkv, cfg.d, cfg.scale, int(cfg.causal), dt,
                                  stream.cuda_stream)
            if st != fb.FA_OK:
                raise RuntimeError(fb.fa_status_string(st))

        ms = time_it(vbwd, 10)
        emit(cfg.name, "bwd", ms, 2.5 * flops, nbytes + 2 * (do.numel() + q.numel() + k.numel() + v.numel()),
             cfg.d)


def sweep_decode(cfg, page, inputs, fb, torch, stream, time_it, emit):
    """Decode against a key/value cache, split over the keys (split kernel + merge kernel)."""
    di = inputs.make_decode(cfg, page_size=page)
    q = di.q.cuda()
    B, Nq, Hq, d = q.shape
    Hkv = di.k.shape[2]
    lens = di.seqlens if di.seqlens is not None else [cfg.Nk] * B
    sl = None if di.seqlens is None else torch.tensor(di.seqlens, dtype=torch.int32, device="cuda")
    ws = torch.empty(fb.fa_decode_workspace_size(B, Hq, Hkv, Nq, d), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    if page:
        kp, vp, bt = di.k_pages.cuda(), di.v_pages.cuda(), di.block_table.cuda()

        def dec():
            st = fb.fa_decode_paged(q.data_ptr(), kp.data_ptr(), vp.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    sl.data_ptr(), bt.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, kp.shape[0],
                                    page, bt.shape[1], d, cfg.scale, int(cfg.causal), dt, stream.cuda_stream)
            if st != fb.FA_OK:
                raise RuntimeError(fb.fa_status_string(st))
    else:
        kc, vc = di.k.cuda(), di.v.cuda()

        def dec():
            st = fb.fa_decode(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              0 if sl is None else sl.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, cfg.Nk, d,
                              cfg.scale, int(cfg.causal), dt, stream.cuda_stream)
            if st != fb.FA_OK:
                raise RuntimeError(fb.fa_status_string(st))

    keys = sum(lens)
    # attention FLOPs (masked pairs of the causal tokens excluded) and the bytes the
    # step must move: every cached K and V row once, Q, O and L
    vis = sum(min(n, max(0, t + n - Nq + 1)) if cfg.causal else n for n in lens for t in range(Nq))
    flops = 4.0 * d * Hq * vis
    nbytes = 2 * (2 * keys * Hkv * d + 2 * q.numel()) + 4 * lse.numel()
    emit(cfg.name + (f"_paged{page}" if page else ""), "decode", time_it(dec, 50), flops, nbytes, d)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave out the per-workload `configs` object of the bench line")
    ap.add_argument("--profile-small", action="store_true",
                    help="run only the warm-up steps on a smaller case (B=1, N=4096) for ncu captures")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                    help="run a few forward calls of one short-sequence workload at full size, or forward + "
                         "backward calls of a small prefill case (for ncu captures)")
    ap.add_argument("--all-configs", action="store_true",
                    help="time the forward of every workload (and the causal GQA backward); one JSON line each")
    ap.add_argument("--only", default=None,
                    help="with --all-configs: only the workload groups whose name contains this text "
                         "(e.g. decode, fp8, window, varlen)")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case(args.profile_case)
    if args.all_configs:
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
