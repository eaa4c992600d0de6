"""Benchmark of the Universal Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one UA prefill forward (token preparation, decay boundary pass, fused biased
attention) over the 1B-shaped workload B=8, T=4096, H=32, Hkv=8, d=64 in bf16, inputs
resident in HBM (they total ~335 MB, larger than the 126 MB L2, so no flush is needed).
`value` is whole-job algorithmic TFLOP/s, F = B*T(T+1)/2*(H*4d + Hkv*2d) per step and GPU.
The line also carries the decode workload (B=32, 16k prefill, 256 steps at p=0.15 and 0.05,
tokens/s and HBM GB/s), the roofline of the dominant kernel, an end-to-end number through
the public API with host buffers, and the fp64 oracle timed on the host cores.

Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no collective on the
data path); time is the max over ranks.  --impl reference times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_compression_ua_b200 import dist  # noqa: E402
from kv_cache_compression_ua_b200 import inputs as I  # noqa: E402

METRIC = "UA prefill TFLOP/s & decode tok/s; % of BF16 TC peak / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

MUFU_PER_CLK_SM = 16   # transcendental (exp2/log2) results per clock per SM: 4 per SM sub-partition
# DRAM bytes (read + written) per launch of the dominant kernel, from the ncu capture summarised
# in profiles/k_fwd_tc_prefill_1b.md; valid only for the kernel version that capture was taken of
TRAFFIC_BYTES = {"k_fwd_tc": 922.77e6 + 149.78e6}   # ncu dram bytes read + written of one launch
N_SM = 148


def mufu_ops(w) -> float:
    """Algorithmic transcendental ops of the bf16 forward: per causal (i, j) pair, 3 per KV head
    for the decay element and 1 per query head for the softmax numerator."""
    return w.B * w.T * (w.T + 1) / 2 * (3 * w.Hkv + w.H)


def fwd_flops(w) -> float:
    """Algorithmic forward FLOPs, counted once: per causal (i, j) pair and batch, H*4d for
    QK^T and PV of every query head plus Hkv*2d for the key-key similarity."""
    return w.B * w.T * (w.T + 1) / 2 * (w.H * 4 * w.d + w.Hkv * 2 * w.d)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clocks and throttle reasons sampled during a region: through NVML every 2 ms when the
    library is there (a short timed region still gets dozens of samples), else nvidia-smi every
    200 ms."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.nvml = None
        self.stop = threading.Event()

    def _nvml_loop(self):
        import pynvml as N
        h = N.nvmlDeviceGetHandleByIndex(self.gpu)
        mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        bits = [0x8, 0x40, 0x20, 0x4]   # hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
        while not self.stop.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                r = N.nvmlDeviceGetCurrentClocksEventReasons(h) if hasattr(
                    N, "nvmlDeviceGetCurrentClocksEventReasons") else N.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                flags = ["Active" if r & b else "Not Active" for b in bits]
                self.lines.append(", ".join([str(sm), str(mx), "0"] + flags))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = threading.Thread(target=self._nvml_loop, daemon=True)
            self.nvml.start()
            time.sleep(0.02)
            return self
        except Exception:
            self.nvml = None
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.nvml is not None:
            time.sleep(0.01)
            self.stop.set()
            self.nvml.join(timeout=5)
            return
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml, 2 ms" if self.nvml is not None else "nvidia-smi, 200 ms"}


# ----------------------------------------------------------------------------- oracle (CPU)

def cpu_model() -> str:
    """The host CPU's model name (for the CPU-baseline record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_sample(w, n_units: int, nthreads: int):
    """Time the fp64 oracle on n_units (batch, KV-head) units of workload w at full T, all
    rows and heads; returns (seconds, algorithmic FLOPs of the sample, description)."""
    import oracle
    b_needed = max(1, math.ceil(n_units / w.Hkv))
    x = I.make_prefill_inputs(w, B=b_needed)
    um = np.zeros(b_needed * w.Hkv, np.uint8)
    um[:n_units] = 1
    oracle._load()
    t0 = time.perf_counter()
    oracle.prefill_fwd(**{k: v for k, v in x.items() if k != "d_o"}, scale=w.scale, theta=w.theta,
                       unit_mask=um, nthreads=nthreads)
    dt = time.perf_counter() - t0
    flops = n_units * w.T * (w.T + 1) / 2 * (w.G * 4 * w.d + 2 * w.d)
    desc = (f"{n_units} of the {w.B * w.Hkv} (batch, KV-head) units of {w.name} at full T={w.T}, "
            f"all rows and {w.G} query heads each, fp64, {nthreads} threads")
    return dt, flops, desc


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = I.WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    n_units = cores
    times = []
    flops = None
    desc = None
    for it in range(args.warmup + args.steps):
        dt, flops, desc = oracle_sample(w, n_units, cores)
        if it >= args.warmup:
            times.append(dt)
    tot = sum(times)
    val = flops * len(times) / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"kind": "oracle", "cores": cores, "cpu_model": cpu_model(), "sample": desc,
                             "value": val, "unit": "TFLOP/s"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w):
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "Hkv": w.Hkv, "head_dim": w.d,
            "dtype": w.dtype, "rope_theta": w.theta, "l2": "inputs (~335 MB) larger than the 126 MB L2, no flush",
            "parallelism": "weak: one batch per GPU"}


# ----------------------------------------------------------------------------- our arm

def device_inputs(w, rank):
    wr = w.resized(seed=dist.rank_seed(w.seed, rank))
    return I.make_prefill_inputs_torch(wr, "cuda")


def bench_prefill(args, world, rank, local, peaks, peaks_kind):
    from kv_cache_compression_ua_b200 import ua
    w = I.WORKLOADS[args.workload]
    x = device_inputs(w, rank)
    out = torch.empty_like(x["q"])
    shape = ua.make_shape(x["q"], x["k"], w.scale, w.theta)
    ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device="cuda")
    bfin = torch.empty(w.B, w.Hkv, w.T, dtype=torch.float32, device="cuda")

    def step():
        # the whole forward contract: O, the row normalisers (for a backward) and b_final (the
        # initial biases of the self-pruning cache)
        ua.prefill_fwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"],
                       scale=w.scale, theta=w.theta, out=out, lse=lse, b_final=bfin, ws=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier(world)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ua.profile_reset()
    ua.profile_enable(True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    ua.profile_enable(False)
    dist.barrier(world)
    tiles, skipped = ua.prefill_tile_stats(shape, ws)
    ms = ev0.elapsed_time(ev1)
    ms_max = dist.max_over_ranks(ms, world)
    prof = ua.profile_read()
    assert ua.get_device_status() == 0
    F = fwd_flops(w)
    value = F * world * args.steps / (ms_max * 1e-3) / 1e12

    # dominant kernel roofline (algorithmic work per launch / measured launch duration)
    top = max(prof.items(), key=lambda kv: kv[1][1])
    name, (launches, tot_ms) = top
    per_launch_ms = tot_ms / launches
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # Tiles whose probabilities all underflow skip their QK^T and PV products (an exactly zero
    # contribution).  `achieved` counts the algorithmic work of the launch (the whole causal
    # triangle), `executed` what the kernel evaluated.
    f_skip = skipped * 128 * 128 * (w.H // w.Hkv) * 4 * w.d
    achieved_t = F / (per_launch_ms * 1e-3) / 1e12
    exec_t = (F - f_skip) / (per_launch_ms * 1e-3) / 1e12
    tensor = {"achieved": achieved_t, "peak": peak_t, "unit": "TFLOP/s", "frac": achieved_t / peak_t,
              "executed": {"achieved": exec_t, "frac": exec_t / peak_t},
              "peak_source": f"{peaks_kind} bf16 burst (MEASURED_PEAKS.json)" if peaks_kind == "measured"
              else "fallback 1590 TF/s"}
    clocks = clk.summary()
    if name == "k_fwd_tc":
        # The fused forward is bound by the exp2/log2 unit, not the tensor pipe: each causal
        # (i, j) pair of a KV head needs 3 transcendental ops for the decay element (softplus:
        # exp and log; cube root: exp of a third of the log) and 1 exp per query head for P.
        mhz = clocks.get("sm_mhz") or 1965.0
        peak_a = MUFU_PER_CLK_SM * N_SM * mhz * 1e6 / 1e9
        # algorithmic transcendental ops of the launch; the executed ones leave out the softmax
        # exps of skipped tiles
        achieved_a = mufu_ops(w) / (per_launch_ms * 1e-3) / 1e9
        exec_a = (mufu_ops(w) - skipped * 128 * 128 * (w.H // w.Hkv)) / (per_launch_ms * 1e-3) / 1e9
        roofline = {"kernel": name, "bound": "alu", "achieved": achieved_a, "peak": peak_a,
                    "unit": "Gop/s (exp2/log2)", "frac": achieved_a / peak_a,
                    "executed": {"achieved": exec_a, "frac": exec_a / peak_a},
                    "traffic": TRAFFIC_BYTES.get(name) if w.name == "prefill_1b" else None,
                    "peak_source": f"{MUFU_PER_CLK_SM} exp2/log2 results per clock per SM x {N_SM} SMs x "
                                   f"{mhz:.0f} MHz (median SM clock sampled during the timed region)",
                    "tensor": tensor}
    else:
        roofline = {"kernel": name, "bound": "tensor", "achieved": achieved_t, "peak": peak_t,
                    "unit": "TFLOP/s", "frac": achieved_t / peak_t, "traffic": None,
                    "peak_source": tensor["peak_source"]}
    roofline.update({"per_launch_ms": per_launch_ms, "share_of_step": tot_ms / sum(v[1] for v in prof.values())})
    roofline["tiles"] = {"causal": tiles, "softmax_skipped": skipped,
                         "executed_tflops": (F - f_skip) * world * args.steps / (ms_max * 1e-3) / 1e12}
    kernels = {k: {"launches": v[0], "total_ms": v[1], "ms_per_launch": v[1] / v[0]} for k, v in prof.items()}
    gpu_launches = sum(v[0] for v in prof.values())
    return w, x, value, ms_max / args.steps, roofline, kernels, gpu_launches, clocks, step


def bench_e2e(args, w, x):
    """Public API with host buffers: every step copies its inputs in from pinned host memory,
    runs the prefill and copies its outputs (O, lse, b_final) out.  Steps are pipelined the way a serving loop would run
    them: two device buffer sets and three streams (copy in, compute, copy out), so step n's
    inputs travel while step n-1 computes and step n-2's output travels back."""
    from kv_cache_compression_ua_b200 import ua
    host = {n: t.cpu().pin_memory() for n, t in x.items()}
    dev = [{n: torch.empty_like(t) for n, t in x.items()} for _ in range(2)]
    out = [torch.empty_like(x["q"]) for _ in range(2)]
    lse = [torch.empty(w.B, w.H, w.T, dtype=torch.float32, device="cuda") for _ in range(2)]
    bfin = [torch.empty(w.B, w.Hkv, w.T, dtype=torch.float32, device="cuda") for _ in range(2)]
    o_host = [torch.empty(x["q"].shape, dtype=x["q"].dtype).pin_memory() for _ in range(2)]
    lse_host = [torch.empty(lse[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    bfin_host = [torch.empty(bfin[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    shape = ua.make_shape(x["q"], x["k"], w.scale, w.theta)
    ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t[0].numel() * t[0].element_size() for t in (o_host, lse_host, bfin_host))
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]      # inputs of buffer set i are on the device
    run_done = [ev(), ev()]     # the prefill that read set i (and wrote out[i]) finished
    out_done = [ev(), ev()]     # out[i] is back on the host
    for e in run_done + out_done:
        e.record(torch.cuda.current_stream())

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(run_done[b])                 # set b is no longer being read
            for n in host:
                dev[b][n].copy_(host[n], non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(in_done[b])
            s_run.wait_event(out_done[b])                # out[b] has been copied back
            d = dev[b]
            ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                           scale=w.scale, theta=w.theta, out=out[b], lse=lse[b], b_final=bfin[b], ws=ws,
                           stream=s_run)
            run_done[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(run_done[b])
            o_host[b].copy_(out[b], non_blocking=True)
            lse_host[b].copy_(lse[b], non_blocking=True)
            bfin_host[b].copy_(bfin[b], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    n = max(4, min(args.steps, 12))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        step(i)
    for st in (s_in, s_run):
        s_out.wait_stream(st)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    return {"value": fwd_flops(w) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "pipelining": "2 buffer sets, copy-in / compute / copy-out streams"}


DECODE_COMPACT_EVERY = 32


def graph_time(run, restore, reps=5, warm=3):
    """Median device time (ms) of `run` captured in one CUDA graph and replayed, the state put
    back by `restore` before every replay (untimed)."""
    g = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_cap):
        run(s_cap)               # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s_cap)
    torch.cuda.synchronize()
    restore()
    with torch.cuda.graph(g, stream=s_cap):
        run(s_cap)
    times = []
    for it in range(warm + reps):
        restore()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        if it >= warm:
            times.append(e0.elapsed_time(e1))
    del g
    return statistics.median(times)


def bench_decode(args, peaks, peaks_kind):
    """Decode workload: B=32 caches prefilled (on the GPU) from a 16k-token draw, compacted at
    p, then 256 single-token steps captured in one CUDA graph and replayed.  Besides the
    workload's thresholds, two supplementary cases: p = 0 (no eviction, the longest caches)
    and a retention-matched draw (the slow mode of a_k moved so that the prefill keeps the
    pages' 16k average share of the keys, 1/21.38 at p = 0.15)."""
    from kv_cache_compression_ua_b200 import ua
    w = I.WORKLOADS["decode_1b"]
    if getattr(args, "decode_batch", None):
        w = w.resized(B=args.decode_batch)         # fewer sequences (profiling captures)
    steps = I.DECODE_STEPS
    T0 = w.T
    x = I.make_prefill_inputs_torch(w, "cuda", names=["k", "v", "a_q", "a_k", "alpha", "beta"])
    q0 = torch.zeros(w.B, T0, w.H, w.d, dtype=torch.bfloat16, device="cuda")
    r = ua.prefill_fwd(q0, x["k"], x["v"], q0, x["a_q"], x["a_k"], x["alpha"], x["beta"],
                       scale=w.scale, theta=w.theta, want_lse=False)
    bfinal = r["b_final"]
    del r
    # Supplementary retention-matched workload: the same draws with the slow mode of a_k moved
    # so that the cache kept after the prefill holds the pages' 16k average share of the keys.
    retained = args.decode_p is None
    if retained:
        wr = w.resized(ak_slow_mean=I.DECODE_RETAINED_AK_SLOW_MEAN)
        ak_r = I.make_prefill_inputs_torch(wr, "cuda", names=["a_k"])["a_k"]
        r = ua.prefill_fwd(q0, x["k"], x["v"], q0, x["a_q"], ak_r, x["alpha"], x["beta"],
                           scale=w.scale, theta=w.theta, want_lse=False)
        bfinal_r = r["b_final"]
        del r
    del q0
    torch.cuda.empty_cache()
    toks = [I.make_decode_token(w, s) for s in range(steps)]
    tok = {n: torch.from_numpy(np.stack([t[n] for t in toks])).to("cuda").to(
        torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32).contiguous() for n in toks[0]}
    ps = list(I.DECODE_THRESHOLDS) + [0.0] if args.decode_p is None else [args.decode_p]
    configs = [(f"p={p:g}" if p > 0 else "p=0 (no eviction, supplementary)", p, x["a_k"], bfinal, tok)
               for p in ps]
    if retained:
        tok_r = dict(tok)
        tok_r["a_k"] = torch.from_numpy(np.stack([I.make_decode_token(wr, s)["a_k"] for s in range(steps)])).to(
            "cuda").to(torch.float32).contiguous()
        configs.append((f"p={I.DECODE_RETAINED_P:g}, retention-matched (supplementary)", I.DECODE_RETAINED_P,
                        ak_r, bfinal_r, tok_r))
    res = {}
    cap = T0 + steps + 1
    entry_bytes = 2 * w.d * 2 + 12          # khat, v (bf16), bias, rk, pos: 268 B at d = 64
    for key, p, ak, bf, tk in configs:
        cache = ua.Cache.empty(w.B, w.Hkv, w.d, cap, torch.bfloat16)
        ua.cache_fill(cache, x["k"], x["v"], ak, bf, theta=w.theta)
        ua.cache_compact(cache, p)
        snap = {n: getattr(cache, n).clone() for n in ("khat", "v", "bias", "rk", "pos", "n_kept")}
        n0 = cache.n_kept.clone()
        o = torch.empty(steps, w.B, w.H, w.d, dtype=torch.bfloat16, device="cuda")

        def restore():
            for n, t in snap.items():
                getattr(cache, n).copy_(t)

        def run_all(stream=None):
            for s in range(steps):
                ua.decode_step(cache, tk["q"][s], tk["k"][s], tk["v"][s], tk["g"][s], tk["a_q"][s],
                               tk["a_k"][s], x["alpha"], x["beta"], T0 + s, p, scale=w.scale, theta=w.theta,
                               out=o[s], stream=stream)

        # kept counts per step (for the byte count): one eager pass
        counts = [n0.sum().item()]
        for s in range(steps):
            ua.decode_step(cache, tk["q"][s], tk["k"][s], tk["v"][s], tk["g"][s], tk["a_q"][s],
                           tk["a_k"][s], x["alpha"], x["beta"], T0 + s, p, scale=w.scale, theta=w.theta,
                           out=o[s])
            counts.append(cache.n_kept.sum().item())
        assert ua.get_device_status() == 0
        final_kept = counts[-1]
        restore()
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_cap):
            run_all(s_cap)           # warm-up on the capture stream
        torch.cuda.current_stream().wait_stream(s_cap)
        torch.cuda.synchronize()
        restore()
        with torch.cuda.graph(g, stream=s_cap):
            run_all(s_cap)
        times = []
        for it in range(3 + 5):
            restore()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        # algorithmic bytes: every live entry read once per step (khat, v, bias, rk, pos), its
        # bias written back, the appended token written, and the token's q/k/v/g/o
        tok_bytes = w.B * (3 * w.H * w.d * 2 + 2 * w.Hkv * w.d * 2 + 2 * w.Hkv * 4)
        bytes_total = sum(counts[s] * entry_bytes + counts[s + 1] * 4 + w.B * w.Hkv * entry_bytes + tok_bytes
                          for s in range(steps))
        gbs = bytes_total / (ms * 1e-3) / 1e9
        kept_frac = final_kept / (w.B * w.Hkv * (T0 + steps))
        res[key] = {"tokens_per_s": w.B * steps / (ms * 1e-3), "ms_per_256_steps": ms,
                    "us_per_step": 1e3 * ms / steps, "hbm_gbs": gbs,
                    "hbm_frac": gbs / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                    "retained_fraction": kept_frac, "kept_entries_after": final_kept,
                    "mean_kept_per_head": float(np.mean(counts)) / (w.B * w.Hkv),
                    "cache_MB_after": final_kept * entry_bytes / 1e6,
                    "compression_x": 1.0 / kept_frac if kept_frac > 0 else None}
        if ak is not x["a_k"]:
            res[key]["ak_slow_mean"] = I.DECODE_RETAINED_AK_SLOW_MEAN
        del g
        if p > 0 and ak is x["a_k"]:
            res[key]["paged"] = bench_decode_paged(w, cache, snap, tk, x, T0, steps, p, o, restore)
        # the same steps through the split walk (deferred compaction; at p > 0 a compaction every
        # DECODE_COMPACT_EVERY steps and after the last), checked against the eager outputs
        ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda")
        o_eager = o.clone()

        def run_split(stream=None):
            for s in range(steps):
                ua.decode_step(cache, tk["q"][s], tk["k"][s], tk["v"][s], tk["g"][s], tk["a_q"][s],
                               tk["a_k"][s], x["alpha"], x["beta"], T0 + s, p, scale=w.scale, theta=w.theta,
                               out=o[s], ws=ws, stream=stream)
                if p > 0 and ((s + 1) % DECODE_COMPACT_EVERY == 0 or s == steps - 1):
                    ua.cache_compact(cache, p, stream=stream)
        restore()
        ms_split = graph_time(run_split, restore)
        assert ua.get_device_status() == 0
        diff = float((o.float() - o_eager.float()).norm() / o_eager.float().norm())
        gbs_s = bytes_total / (ms_split * 1e-3) / 1e9
        res[key]["split_walk"] = {
            "us_per_step": 1e3 * ms_split / steps, "tokens_per_s": w.B * steps / (ms_split * 1e-3),
            "hbm_gbs": gbs_s, "hbm_frac": gbs_s / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
            "compaction": (f"deferred, every {DECODE_COMPACT_EVERY} steps" if p > 0 else "none needed (p = 0)"),
            "o_rel_l2_vs_one_cta_per_cache": diff}
        del cache, snap, ws
        torch.cuda.empty_cache()
    # Split walk for few long caches (supplementary): one sequence (B=1, 8 KV heads, p = 0: 16.4k
    # live pairs per head, compaction deferred) decoded by one CTA per cache and by the split step
    # (up to 16 CTAs per cache), both graph-captured.
    xs = {n: x[n][:1].contiguous() for n in ("k", "v", "a_k")}
    bf1 = bfinal[:1].contiguous()
    tk1 = {n: t[:, :1].contiguous() for n, t in tok.items()}
    split_res = {}
    for mode in ("one CTA per cache", "split"):
        cache = ua.Cache.empty(1, w.Hkv, w.d, cap, torch.bfloat16)
        ua.cache_fill(cache, xs["k"], xs["v"], xs["a_k"], bf1, theta=w.theta)
        ua.cache_compact(cache, 0.0)
        snap = {n: getattr(cache, n).clone() for n in ("khat", "v", "bias", "rk", "pos", "n_kept")}
        n0 = int(cache.n_kept.sum().item())
        o = torch.empty(steps, 1, w.H, w.d, dtype=torch.bfloat16, device="cuda")
        ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda") if mode == "split" else None

        def run1(stream=None):
            for s in range(steps):
                ua.decode_step(cache, tk1["q"][s], tk1["k"][s], tk1["v"][s], tk1["g"][s], tk1["a_q"][s],
                               tk1["a_k"][s], x["alpha"], x["beta"], T0 + s, 0.0, scale=w.scale, theta=w.theta,
                               out=o[s], defer_compact=True, ws=ws, stream=stream)

        def restore1():
            for n, t in snap.items():
                getattr(cache, n).copy_(t)
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_cap):
            run1(s_cap)
        torch.cuda.current_stream().wait_stream(s_cap)
        torch.cuda.synchronize()
        restore1()
        with torch.cuda.graph(g, stream=s_cap):
            run1(s_cap)
        times = []
        for it in range(3 + 5):
            restore1()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
        assert ua.get_device_status() == 0
        ms = statistics.median(times)
        byts = sum((n0 + w.Hkv * s) * entry_bytes + (n0 + w.Hkv * (s + 1)) * 4 for s in range(steps))
        split_res[mode] = {"us_per_step": 1e3 * ms / steps, "tokens_per_s": steps / (ms * 1e-3),
                           "hbm_gbs": byts / (ms * 1e-3) / 1e9,
                           "hbm_frac": byts / (ms * 1e-3) / 1e9 / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])}
        del g, cache, snap
        torch.cuda.empty_cache()
    split_res["workload"] = (f"decode_1b batch 0 only: B=1, {w.Hkv} KV heads, p=0 (16.4k live pairs per head), "
                             f"{steps} steps, deferred compaction, graph-captured")
    res["few_long_caches (supplementary)"] = split_res
    res["peak_source"] = f"{peaks_kind} HBM copy bandwidth"
    res["workload"] = f"decode_1b: B={w.B}, 16k prefill, {steps} steps, graph-captured"
    return res


def bench_decode_paged(w, cache, snap, tk, x, T0, steps, p, o_ref, restore_ref):
    """The same graph-replayed eager steps on paged storage: the compacted caches' live pairs moved
    to a pool of 128-slot pages that holds them and the appends of the coming steps only (pages for
    the appends are given before capture, as a graph cannot call the host allocator between
    steps).  Reports the step time and the pool's size against the contiguous caches'."""
    from kv_cache_compression_ua_b200 import ua
    ps = 128
    restore_ref()
    n0 = cache.n_kept.reshape(-1).cpu().numpy().astype(np.int64)
    need = (n0 + steps + ps - 1) // ps
    max_pages = (cache.capacity + ps - 1) // ps
    paged = ua.Cache.paged(w.B, w.Hkv, w.d, ps, max_pages, int(need.sum()), torch.bfloat16)
    pool = ua.PagePool(paged)
    pool.ensure(n0 + steps)
    # move the live pairs (setup, not timed)
    tab = paged.page_table.long()
    for u in range(w.B * w.Hkv):
        n = int(n0[u])
        if n == 0:
            continue
        s_idx = torch.arange(n, device="cuda")
        dst = tab[u, s_idx // ps] * ps + s_idx % ps
        b, h = divmod(u, w.Hkv)
        for name in ("khat", "v", "bias", "rk", "pos"):
            getattr(paged, name)[dst] = getattr(cache, name)[b, h, :n]
    paged.n_kept.copy_(cache.n_kept)
    psnap = {n: getattr(paged, n).clone() for n in ("khat", "v", "bias", "rk", "pos", "n_kept")}
    o = torch.empty_like(o_ref)

    def restore():
        for n, t in psnap.items():
            getattr(paged, n).copy_(t)

    def run_all(stream=None):
        for s in range(steps):
            ua.decode_step(paged, tk["q"][s], tk["k"][s], tk["v"][s], tk["g"][s], tk["a_q"][s], tk["a_k"][s],
                           x["alpha"], x["beta"], T0 + s, p, scale=w.scale, theta=w.theta, out=o[s], stream=stream)
    restore()
    run_all()
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    same = bool(torch.equal(o, o_ref))
    ms = graph_time(run_all, restore)
    entry = 2 * w.d * 2 + 12
    return {"us_per_step": 1e3 * ms / steps, "page_slots": ps, "pages": int(need.sum()),
            "pool_MB": int(need.sum()) * ps * entry / 1e6,
            "contiguous_MB": w.B * w.Hkv * cache.capacity * entry / 1e6,
            "outputs_identical_to_contiguous": same}


def time_prefill(w, x, steps, warmup, prune_p=0.0, want_bfinal=True):
    """Device time of `steps` prefill forwards of workload w (inputs x resident in HBM), with the
    per-kernel launch times and the tile statistics of the last call."""
    from kv_cache_compression_ua_b200 import ua
    out = torch.empty_like(x["q"])
    shape = ua.make_shape(x["q"], x["k"], w.scale, w.theta, prune_p=prune_p)
    ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device="cuda")
    bfin = torch.empty(w.B, w.Hkv, w.T, dtype=torch.float32, device="cuda") if want_bfinal else None

    def step():
        ua.prefill_fwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"],
                       scale=w.scale, theta=w.theta, out=out, lse=lse, b_final=bfin, want_bfinal=want_bfinal,
                       ws=ws, prune_p=prune_p)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ua.profile_reset()
    ua.profile_enable(True)
    ev0.record()
    for _ in range(steps):
        step()
    ev1.record()
    torch.cuda.synchronize()
    ua.profile_enable(False)
    prof = ua.profile_read()
    tiles, skipped = ua.prefill_tile_stats(shape, ws)
    assert ua.get_device_status() == 0
    return ev0.elapsed_time(ev1) / steps, prof, tiles, skipped


def bench_prefill_more(args, peaks, peaks_kind, mhz):
    """The other prefill configurations: the 16k-token long-context prefill (B=1, bimodal a_k,
    b_final emitted), the chunked pruned prefill of the 1B workload at p = 0.05 and 0.15 and of
    the 3B-shaped forward (head_dim 128) at p = 0.15 (128-token chunks), each with the roofline
    of its fused kernel where it is the head_dim-64 one."""
    res = {}
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_a = MUFU_PER_CLK_SM * N_SM * (mhz or 1965.0) * 1e6 / 1e9
    cases = [("prefill_1b_16k", 0.0)] + [("prefill_1b", p) for p in I.DECODE_THRESHOLDS] + [("fwdbwd_3b", 0.15)]
    for wname, p in cases:
        w = I.WORKLOADS[wname]
        x = I.make_prefill_inputs_torch(w, "cuda")
        steps = max(10, min(args.steps, 50))
        ms, prof, tiles, skipped = time_prefill(w, x, steps, 3, prune_p=p)
        F = fwd_flops(w)
        G = w.H // w.Hkv
        entry = {"workload": f"{wname}: B={w.B} T={w.T} H={w.H} Hkv={w.Hkv} d={w.d} bf16"
                             + (f", chunked pruned prefill p={p:g} (128-token chunks)" if p > 0 else ""),
                 "ms_per_step": ms, "tflops_dense_equiv": F / (ms * 1e-3) / 1e12,
                 "tokens_per_s": w.B * w.T / (ms * 1e-3), "steps": steps,
                 "kernels": {k: {"launches": v[0], "ms_per_launch": v[1] / v[0]} for k, v in prof.items()},
                 "tiles": {"causal": tiles, "softmax_skipped": skipped}}
        if "k_fwd_tc" in prof:
            kms = prof["k_fwd_tc"][1] / prof["k_fwd_tc"][0]
            f_exec = F - skipped * 128 * 128 * G * 4 * w.d
            ops = mufu_ops(w) - skipped * 128 * 128 * G
            # as the headline line: `achieved` the whole causal triangle's algorithmic work,
            # `executed` what ran (with chunked pruning the evicted pairs' softmax is not part of
            # the method's work either, so there the executed figure is the one to read)
            entry["roofline"] = {
                "kernel": "k_fwd_tc", "bound": "alu", "per_launch_ms": kms,
                "achieved": mufu_ops(w) / (kms * 1e-3) / 1e9, "peak": peak_a, "unit": "Gop/s (exp2/log2)",
                "frac": mufu_ops(w) / (kms * 1e-3) / 1e9 / peak_a,
                "executed": {"achieved": ops / (kms * 1e-3) / 1e9, "frac": ops / (kms * 1e-3) / 1e9 / peak_a},
                "tensor": {"achieved": F / (kms * 1e-3) / 1e12, "peak": peak_t, "unit": "TFLOP/s",
                           "frac": F / (kms * 1e-3) / 1e12 / peak_t,
                           "executed": {"achieved": f_exec / (kms * 1e-3) / 1e12,
                                        "frac": f_exec / (kms * 1e-3) / 1e12 / peak_t}}}
        res[("prefill_3b" if wname == "fwdbwd_3b" else wname) + (f"_pruned_p{p:g}" if p > 0 else "")] = entry
        del x
        torch.cuda.empty_cache()
    return res


def bwd_flops(w) -> float:
    """Algorithmic backward FLOPs, counted once: per causal pair and batch, H*10d (the S, dP,
    dV, dK and dQ products of every query head) plus Hkv*6d (the key-key similarity, and its
    two gradient products)."""
    return w.B * w.T * (w.T + 1) / 2 * (w.H * 10 * w.d + w.Hkv * 6 * w.d)


def bench_fwdbwd(args):
    """3B layer forward + backward (B=4, T=8192, H=24, Hkv=8, d=128, bf16)."""
    from kv_cache_compression_ua_b200 import ua
    w = I.WORKLOADS["fwdbwd_3b"]
    if args.fwdbwd_batch != w.B:
        w = w.resized(B=args.fwdbwd_batch)
    x = I.make_prefill_inputs_torch(w, "cuda")
    args_in = (x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    shape = ua.make_shape(x["q"], x["k"], w.scale, w.theta)
    wsf = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    wsb = ua.alloc_workspace(ua.prefill_bwd_workspace_size(shape), "cuda")
    f = ua.prefill_fwd(*args_in, scale=w.scale, theta=w.theta, ws=wsf)
    ua.prefill_bwd(*args_in, f["o"], f["lse"], f["b_final"], x["d_o"], scale=w.scale, theta=w.theta, ws=wsb)
    torch.cuda.synchronize()
    n = 3
    ua.profile_reset()
    ua.profile_enable(True)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record()
    for _ in range(n):
        f = ua.prefill_fwd(*args_in, scale=w.scale, theta=w.theta, ws=wsf)
    e[1].record()
    for _ in range(n):
        ua.prefill_bwd(*args_in, f["o"], f["lse"], f["b_final"], x["d_o"], scale=w.scale, theta=w.theta, ws=wsb)
    e[2].record()
    torch.cuda.synchronize()
    ua.profile_enable(False)
    prof = ua.profile_read()
    assert ua.get_device_status() == 0
    fms, bms = e[0].elapsed_time(e[1]) / n, e[1].elapsed_time(e[2]) / n
    steps, walked = ua.prefill_bwd_band_stats(shape, wsb)
    band = {"steps": steps, "walked": walked, "walked_fraction": walked / steps,
            "bwd_tflops_walked_estimate": bwd_flops(w) * walked / steps / (bms * 1e-3) / 1e12}
    return {"workload": f"fwdbwd_3b: B={w.B} T={w.T} H={w.H} Hkv={w.Hkv} d={w.d} bf16", "fwd_ms": fms, "bwd_ms": bms,
            "bwd_band": band,
            "fwd_tflops": fwd_flops(w) / (fms * 1e-3) / 1e12, "bwd_tflops": bwd_flops(w) / (bms * 1e-3) / 1e12,
            "fwd_bwd_tflops": (fwd_flops(w) + bwd_flops(w)) / ((fms + bms) * 1e-3) / 1e12,
            "flops_basis": "dense-equivalent: the whole causal triangle's FLOPs; both passes skip exactly "
                           "underflowing tiles (the forward its softmax, the backward the band below each "
                           "key tile's last step with a possibly nonzero probability)",
            "kernels": {k: {"launches": v[0], "ms_per_launch": v[1] / v[0]} for k, v in prof.items()}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_1b")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-more", action="store_true", help="skip the 16k and chunked-pruned prefill lines")
    ap.add_argument("--decode-p", type=float, default=None, help="run the decode section at this p only")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="sequences of the decode section (default: the workload's 32; smaller for profiling)")
    ap.add_argument("--fwdbwd-batch", type=int, default=4,
                    help="batch of the 3B forward+backward line (4 = the workload; smaller for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist.init("nccl") if args.impl == "ours" else dist.env_world()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    from kv_cache_compression_ua_b200 import build as ua_build
    if rank == 0 and not os.path.exists(os.path.join(ROOT, "kv_cache_compression_ua_b200", "libua.so")):
        ua_build.build()
    dist.barrier(world)
    peaks, peaks_kind = load_peaks()
    w, x, value, ms_step, roofline, kernels, launches, clocks, _ = bench_prefill(
        args, world, rank, local, peaks, peaks_kind)
    e2e = bench_e2e(args, w, x)
    del x
    torch.cuda.empty_cache()
    decode = None
    if not args.no_decode and world == 1:
        decode = bench_decode(args, peaks, peaks_kind)
    more = None
    if not args.no_more and world == 1:
        more = bench_prefill_more(args, peaks, peaks_kind, clocks.get("sm_mhz"))
    fwdbwd = None
    if not args.no_bwd and world == 1:
        torch.cuda.empty_cache()
        fwdbwd = bench_fwdbwd(args)
    cpu = None
    if not args.no_cpu and rank == 0 and world == 1:
        cores = os.cpu_count() or 1
        dt, fl, desc = oracle_sample(w, cores, cores)
        dt1, fl1, desc1 = oracle_sample(w, 1, 1)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
               "sample": desc, "seconds": dt,
               "single_core": {"value": fl1 / dt1 / 1e12, "unit": "TFLOP/s", "sample": desc1, "seconds": dt1}}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": workload_config(w), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clocks, "kernels": kernels, "prefill_more": more,
                "decode": decode, "fwdbwd_3b": fwdbwd}
        print(json.dumps(line), flush=True)
    dist.finalize(world)


if __name__ == "__main__":
    main()
