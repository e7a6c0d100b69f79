"""Benchmark of the MoE layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, top-k, count/scan/permute, grouped
expert FFN, combine, balance statistics) through moe_forward on one batch of
synthetic input already resident in HBM.  The default workload is the
Qwen3-MoE-shaped layer (T=16384, d_model=2048, 128 experts of d_ff=768, top-8,
Zipf(1.1) expert popularity).  Under torchrun every rank runs an independent
replica (the layer forward has no data-path exchange), so `value` is the sum
of tokens over ranks divided by the slowest rank's time ("weak" scaling).

--impl reference times the CPU oracle (fp64, host cores) on a bounded sample
of the same workload; under torchrun only rank 0 runs it.
"""
import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_49_b200 import native as nat  # noqa: E402
from mixture_experts_layer_49_b200 import synthetic as syn  # noqa: E402

METRIC = "MoE-layer fwd tokens/s and % of roofline (tensor or HBM) on 1 B200"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------- util
def max_over_ranks(values, world, device):
    """Per-rank timings reduced to the slowest rank's (all_reduce MAX); with
    one rank, the values themselves."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(world, T, ms):
    """Whole-job throughput: every rank runs a replica on its own T tokens, so
    the job moves world * T tokens per step of the slowest rank."""
    return world * T / (ms * 1e-3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling around the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        power = [float(r[3]) for r in rows if re.match(r"^[0-9.]+$", r[3])]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


def source_hash(path):
    """sha256 (first 12 hex digits) of a source file with its comments, trailing
    blanks and blank lines removed: a comment edit keeps the hash, any change to
    the code changes it."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines()]
    code = "\n".join(ln for ln in lines if ln)
    return hashlib.sha256(code.encode()).hexdigest()[:12]


def recorded_traffic(workload, kernel="grouped_ffn"):
    """DRAM bytes per launch of the grouped-FFN kernels (kernel: grouped_ffn or
    grouped_ffn_fp8) from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    if not os.path.exists(path):
        return None
    src = source_hash(os.path.join(ROOT, "mixture_experts_layer_49_b200", "csrc", "ffn_sm100.cu"))
    for line in open(path):
        m = re.match(r"\|\s*(\w+)\s*\|\s*(\w+)\s*\|\s*([0-9a-f]+)\s*\|\s*([0-9.eE+]+)\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == workload and m.group(3) == src:
            return float(m.group(4))
    return None


def algorithmic_counts(wl, counts, kept, fp8=False):
    """Expert FLOPs on kept rows (+ shared expert), and the layer's algorithmic
    bytes: x, y, W_r and the weights of every expert with a kept row (e4m3
    experts: one byte per weight plus a 4-byte scale per output channel)."""
    esz = 2 if wl.dtype == "bf16" else 4
    wsz = 1 if fp8 else esz
    mats = 3 if wl.act == "swiglu" else 2
    kept_rows = int(kept.sum())
    flops = wl.expert_flops(kept_rows)
    touched = int((kept > 0).sum())
    w_bytes = touched * mats * wl.d_model * wl.d_ff * wsz
    if fp8:                                        # per-channel scales
        w_bytes += touched * 4 * ((mats - 1) * wl.d_ff + wl.d_model)
    if wl.d_ff_shared:
        w_bytes += 3 * wl.d_model * wl.d_ff_shared * wsz
    b = 2 * wl.T * wl.d_model * esz + wl.d_model * wl.E * 4 + w_bytes
    return flops, b, kept_rows


# ------------------------------------------------------------- CPU oracle leg
def oracle_sample(wl, inp_host, target_s, max_tokens=None, threads=None):
    """Time the oracle (router + selection + expert FFNs in fp64) on the first
    n tokens of the workload; n is grown until the run takes ~target_s.
    threads: worker threads (default: every host core)."""
    import oracle
    cap = oracle.capacity(float(np.float32(wl.capacity_factor)), wl.top_k, wl.T, wl.E)
    weights = {k: inp_host[k] for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd")
               if inp_host.get(k) is not None}
    n = 8
    while True:
        dims = oracle.make_dims(n, wl.d_model, wl.E, wl.d_ff, wl.top_k, x_dtype=wl.dtype, act=wl.act,
                                score=wl.score, renorm=wl.renorm, capacity=cap,
                                d_ff_shared=wl.d_ff_shared, nthreads=threads)
        x = inp_host["x"][:n]
        t0 = time.perf_counter()
        r = oracle.route(dims, x, inp_host["Wr"], inp_host["logit_bias"], inp_host["sel_bias"])
        dp = oracle.dispatch(dims, r["idx"])
        oracle.balance(dims, dp["counts"], r["pnorm"])
        oracle.layer_tokens(dims, x, weights, r["idx"], r["gate"], dp["row_of"], np.arange(n, dtype=np.int32))
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or n >= (max_tokens or wl.T):
            return n, dt, dims.nthreads
        n = min(max_tokens or wl.T, max(n * 2, int(n * target_s / max(dt, 1e-3) * 0.8)))


def host_inputs(inp):
    return {k: (syn.to_numpy_raw(v) if isinstance(v, torch.Tensor) else None)
            for k, v in inp.items() if k != "workload"}


def run_reference(args, wl, dev):
    inp = syn.generate(wl, dev, seed=0)
    host = host_inputs(inp)
    del inp
    per_step = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    n, _, cores = oracle_sample(wl, host, per_step)
    import oracle
    cap = oracle.capacity(float(np.float32(wl.capacity_factor)), wl.top_k, wl.T, wl.E)
    dims = oracle.make_dims(n, wl.d_model, wl.E, wl.d_ff, wl.top_k, x_dtype=wl.dtype, act=wl.act,
                            score=wl.score, renorm=wl.renorm, capacity=cap, d_ff_shared=wl.d_ff_shared)
    weights = {k: host[k] for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd") if host.get(k) is not None}

    def step(i):
        lo = (i * n) % max(1, wl.T - n + 1)
        x = np.ascontiguousarray(host["x"][lo:lo + n])
        r = oracle.route(dims, x, host["Wr"], host["logit_bias"], host["sel_bias"])
        dp = oracle.dispatch(dims, r["idx"])
        oracle.balance(dims, dp["counts"], r["pnorm"])
        oracle.layer_tokens(dims, x, weights, r["idx"], r["gate"], dp["row_of"], np.arange(n, dtype=np.int32))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = ("%d consecutive tokens of %s per step (router, top-k, dispatch, balance and expert FFNs "
              "in fp64 for those tokens)" % (n, wl.name))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(workload_config(wl), l2="n/a: host oracle"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(wl):
    return {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "E": wl.E, "d_ff": wl.d_ff,
            "top_k": wl.top_k, "act": wl.act, "score": wl.score, "renorm": wl.renorm,
            "capacity_factor": wl.capacity_factor, "d_ff_shared": wl.d_ff_shared,
            "logit_skew": wl.logit_skew, "l2": "flushed between steps (256 MiB write)",
            "router": "frozen weights (moe_router_freeze: the W_r split once, before timing)"}


# ------------------------------------------------------------------ GPU leg
def run_ours(args, wl, dev, world, rank, fp8=None, steps=None, warmup=None, full=True):
    """Time K whole-layer steps of `wl` (and, with full, the end-to-end leg
    and the CPU baseline).  Sub-records pass full=False: the device-resident
    steps and the staged per-stage pass only."""
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    fp8 = (args.experts == "fp8") if fp8 is None else fp8
    steps = args.steps if steps is None else steps
    warmup = args.warmup if warmup is None else warmup
    inp = syn.generate(wl, dev, seed=0, weights=not fp8)
    w8 = None
    if fp8:                                         # e4m3 experts (bf16 layer around them)
        w8 = syn.generate_fp8_experts(wl, dev, seed=0)
        inp["b1"], inp["b2"] = w8.get("b1"), w8.get("b2")
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, dev)
    ws = nat.alloc_workspace(cfg, dev)
    # the router weights stay fixed while the layer serves: split W_r once (moe_router_freeze)
    nat.moe_router_freeze(cfg, inp["Wr"], ws, stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def layer(inp_, out_):
        if fp8:
            nat.forward_fp8(cfg, inp_, w8, out_, ws, stream)
        else:
            nat.forward(cfg, inp_, out_, ws, stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[dev.index])

    for _ in range(warmup):
        flush.zero_()
        layer(inp, out)
    torch.cuda.synchronize(dev)
    st = nat.moe_get_device_status(ws, stream)
    if st != nat.MOE_OK:
        raise RuntimeError("device status after warm-up: " + nat.status_string(st))

    # ---- main timed region: K whole-layer steps through moe_forward
    sampler = ClockSampler(dev.index)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    barrier()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        layer(inp, out)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = sum(step_ms) / steps
    srt = sorted(step_ms)
    step_pct = {q: srt[min(len(srt) - 1, int(round(q / 100 * (len(srt) - 1))))] for q in (10, 50, 90)}
    st = nat.moe_get_device_status(ws, stream)
    if st != nat.MOE_OK:
        raise RuntimeError("device status after timing: " + nat.status_string(st))

    # ---- per-stage timing through the staged entry points (same kernels)
    T, d, E, k = wl.T, wl.d_model, wl.E, wl.top_k
    dt = nat.layer_dtype(cfg)
    psum = torch.empty((nat.router_blocks(cfg), E), dtype=torch.float32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_gate = torch.empty(T * k, dtype=torch.float32, device=dev)
    x_perm = torch.empty((T * k, d), dtype=torch.uint8 if fp8 else dt, device=dev)
    y_perm = torch.empty((nat.perm_rows(cfg), d), dtype=dt, device=dev)
    if fp8:
        # e4m3 x and its packed rows, built once from this step's routing (the
        # forward quantizes x and copies its rows on the device; here the
        # staged pass times the quantizer, the row tables and the FFN)
        x8 = torch.empty((T, d), dtype=torch.uint8, device=dev)
        xs = torch.empty(T, dtype=torch.float32, device=dev)
        xps = torch.zeros(T * k, dtype=torch.float32, device=dev)
        nat.moe_quantize_rows_e4m3(inp["x"], x8, xs, stream=stream)
        nat.moe_permute(cfg, inp["x"], out.idx, out.gate, out.counts, kept, offsets, row_of, row_token, row_gate,
                        None, out.n_dropped, ws, stream)
        torch.cuda.synchronize(dev)
        nrows = int(offsets[-1].item())
        x_perm[:nrows] = x8[row_token[:nrows].long()]
        xps[:nrows] = xs[row_token[:nrows].long()]
    stages = ["router", "permute", "grouped_ffn", "combine", "balance"]
    stage_ms = {s: [] for s in stages}
    all_evs = []
    for it in range(warmup + steps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        evs[0].record(stream)
        nat.moe_router_topk(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"], out.idx, out.gate,
                            None, psum, ws, stream)
        evs[1].record(stream)
        if fp8:
            nat.moe_quantize_rows_e4m3(inp["x"], x8, xs, stream=stream)
            nat.moe_permute(cfg, inp["x"], out.idx, out.gate, out.counts, kept, offsets, row_of, row_token,
                            row_gate, None, out.n_dropped, ws, stream)
        else:
            nat.moe_permute(cfg, inp["x"], out.idx, out.gate, out.counts, kept, offsets, row_of, row_token,
                            row_gate, x_perm, out.n_dropped, ws, stream)
        evs[2].record(stream)
        if fp8:
            nat.moe_grouped_ffn_fp8(cfg, x_perm, xps, offsets, row_gate, w8, inp["b1"], inp["b2"], x8, xs, y_perm,
                                    ws, stream)
        else:
            nat.moe_grouped_ffn(cfg, x_perm, offsets, row_gate, inp["W1"], inp["b1"], inp["Wu"], inp["W2"],
                                inp["b2"], inp["x"], inp["Wsg"], inp["Wsu"], inp["Wsd"], y_perm, ws, stream)
        evs[3].record(stream)
        nat.moe_combine(cfg, y_perm, row_of, out.y, ws, stream)
        evs[4].record(stream)
        nat.moe_balance_stats(cfg, out.counts, psum, out.f, out.P, out.loss, stream)
        evs[5].record(stream)
        if it >= warmup:
            all_evs.append(evs)
    torch.cuda.synchronize(dev)       # once: the host runs ahead, so no launch gaps land in a stage
    for evs in all_evs:
        for j, name in enumerate(stages):
            stage_ms[name].append(evs[j].elapsed_time(evs[j + 1]))
    stage_avg = {s: sum(v) / len(v) for s, v in stage_ms.items()}

    if not full:
        e2e_ms = float("nan")
        x_host = y_host = None
    else:
        e2e_ms, x_host, y_host = time_e2e(cfg, inp, out, layer, stream, dev, warmup, steps)
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, dev)
    return finish(args, wl, cfg, inp, out, dev, rank, fp8, full, ms, e2e_ms, x_host, y_host, clocks, stage_avg,
                  step_pct)


def time_e2e(cfg, inp, out, layer, stream, dev, warmup, steps):
    # ---- end to end through moe_forward: every step copies its own x in
    # (pinned host -> device) and its y and loss out, all inside the timed
    # region.  Copies run on their own streams with double-buffered device
    # buffers, so step i's input copy and step i-1's output copy overlap step
    # i's layer (the per-step working set, weights and permuted rows, is well
    # above L2, so no flush is needed between steps).
    nbuf = 2
    x_host = inp["x"].cpu().pin_memory()
    y_host = [torch.empty_like(out.y, device="cpu").pin_memory() for _ in range(nbuf)]
    loss_host = [torch.empty(1, dtype=torch.float64).pin_memory() for _ in range(nbuf)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(nbuf)]
    outs = [nat.Outputs(cfg, dev) for _ in range(nbuf)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n_e2e = warmup + steps
    ev_in = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_comp = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_out = [torch.cuda.Event() for _ in range(n_e2e)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    for i in range(n_e2e):
        b = i % nbuf
        if i >= nbuf:
            s_in.wait_event(ev_comp[i - nbuf])       # x_dev[b] is free once its layer ran
        if i == warmup:
            t_start.record(s_in)
        with torch.cuda.stream(s_in):
            x_dev[b].copy_(x_host, non_blocking=True)
        ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if i >= nbuf:
            stream.wait_event(ev_out[i - nbuf])      # outs[b] is free once its results are out
        inp_i = dict(inp)
        inp_i["x"] = x_dev[b]
        layer(inp_i, outs[b])
        ev_comp[i].record(stream)
        s_out.wait_event(ev_comp[i])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(outs[b].y, non_blocking=True)
            loss_host[b].copy_(outs[b].loss, non_blocking=True)
        ev_out[i].record(s_out)
    t_end.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = t_start.elapsed_time(t_end) / steps
    return e2e_ms, x_host, y_host[0]


def tensor_peak(peaks, clocks):
    """The tensor peak a run is held to: the burst figure, unless the clocks
    sampled during that run's timed region show sw_power_cap active, in which
    case the sustained (power-capped) figure.  Returns (TFLOP/s, which)."""
    if "sw_power_cap" in (clocks.get("reasons") or []):
        return peaks["bf16_tflops_sustained"], "sustained (sw_power_cap active during the timed region)"
    return peaks["bf16_tflops"], "burst (no power cap during the timed region)"


def finish(args, wl, cfg, inp, out, dev, rank, fp8, full, ms, e2e_ms, x_host, y_host, clocks, stage_avg, step_pct):
    counts = out.counts.cpu().numpy()
    cap = nat.capacity(cfg)
    kept_np = np.minimum(counts, cap) if cap >= 0 else counts
    flops, alg_bytes, kept_rows = algorithmic_counts(wl, counts, kept_np, fp8)
    peaks, peak_src = load_peaks()
    if fp8:       # e4m3 contractions: the measured bf16 peaks x the nominal fp8 : bf16 ratio (2)
        peaks = dict(peaks, bf16_tflops=2 * peaks["bf16_tflops"],
                     bf16_tflops_sustained=2 * peaks["bf16_tflops_sustained"])
    peak_t, peak_which = tensor_peak(peaks, clocks)
    t_tensor = flops / (peak_t * 1e12)
    t_tensor_burst = flops / (peaks["bf16_tflops"] * 1e12)
    t_tensor_sust = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    ffn_ms = stage_avg["grouped_ffn"]
    ffn_tflops = flops / (ffn_ms * 1e-3) / 1e12
    traffic = recorded_traffic(wl.name, "grouped_ffn_fp8" if fp8 else "grouped_ffn")
    result = dict(rank=rank, ms=ms, e2e_ms=e2e_ms, clocks=clocks, stage_avg=stage_avg, counts=counts, step_pct=step_pct,
                  flops=flops, alg_bytes=alg_bytes, kept_rows=kept_rows, peaks=peaks, peak_src=peak_src,
                  peak_t=peak_t, peak_which=peak_which,
                  layer_roof_ms=max(t_tensor, t_hbm) * 1e3, layer_roof_burst_ms=max(t_tensor_burst, t_hbm) * 1e3,
                  layer_roof_sust_ms=max(t_tensor_sust, t_hbm) * 1e3, ffn_tflops=ffn_tflops,
                  traffic=traffic,
                  loss=float(out.loss.item()), n_dropped=int(out.n_dropped.item()),
                  bound="tensor" if t_tensor >= t_hbm else "hbm")
    if full:
        result["h2d"] = x_host.numel() * x_host.element_size()
        result["d2h"] = y_host.numel() * y_host.element_size() + 8
    if full and rank == 0 and not args.no_cpu_baseline and not fp8:
        host = host_inputs(inp)
        n, dt_cpu, cores = oracle_sample(wl, host, args.cpu_seconds)
        n1, dt1, _ = oracle_sample(wl, host, max(1.0, args.cpu_seconds / 5), threads=1)
        result["cpu"] = {"value": n / dt_cpu, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "first %d tokens of %s: router, top-k, dispatch, balance and expert FFNs in "
                                   "fp64 (%.1f s on the host cores)" % (n, wl.name, dt_cpu),
                         "value_1core": n1 / dt1,
                         "sample_1core": "first %d tokens, one thread (%.1f s)" % (n1, dt1)}
    return result


def launches_per_forward(wl, fp8=False):
    """Kernels one moe_forward call launches (T > 0) on a workspace whose router
    is frozen (moe_router_freeze: the W_r split is done once, before timing).
    bf16: logits GEMM, selection, histogram, scan (+ balance statistics),
    permute, two launches per expert GEMM (CTA-pair kernel, then the 1-CTA
    kernel for last blocks of 1..128 rows), combine.  fp32: router,
    histogram, scan, permute, two SIMT GEMMs, combine.  moe_forward_fp8 adds
    the quantization of x and of H (the routed rows, and the shared rows when
    there is a shared expert)."""
    if fp8:
        return 12 + (1 if wl.d_ff_shared else 0)
    return 10 if wl.dtype == "bf16" else 7


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_moe", choices=sorted(syn.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--experts", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: e4m3 experts through moe_forward_fp8 (bf16 layers only; no CPU baseline)")
    ap.add_argument("--sub", default="mixtral,deepseek_v3,qwen3_moe:fp8,qwen3_moe:mx,qwen3_moe:w4,qwen3_moe:backward",
                    help="further workloads (name or name:fp8) timed after the headline one and reported "
                         "under sub_records; '' for none")
    ap.add_argument("--sub-steps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    wl = syn.WORKLOADS[args.workload]
    if args.experts == "fp8" and wl.dtype != "bf16":
        ap.error("--experts fp8 needs a bf16 workload")
    if args.impl == "reference":
        if rank == 0:
            dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
            run_reference(args, wl, dev)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    subs = {}
    try:
        r = run_ours(args, wl, dev, world, rank)
        for spec in [t for t in args.sub.split(",") if t] if args.experts == "bf16" else []:
            torch.cuda.empty_cache()
            try:
                subs[spec] = sub_record(args, spec, dev, world, rank)
            except Exception as exc:           # a failed sub-record is reported, the headline stands
                subs[spec] = {"error": "%s: %s" % (type(exc).__name__, exc)}
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank != 0:
        return
    tokens_per_s = job_tokens_per_s(world, wl.T, r["ms"])
    e2e_tokens_per_s = job_tokens_per_s(world, wl.T, r["e2e_ms"])
    fp8 = args.experts == "fp8"
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 experts (fp32 accumulation), bf16 layer" if fp8 else ("bf16" if wl.dtype == "bf16"
                                                                                   else "f32"),
        "data": "synthetic",
        "config": dict(workload_config(wl), parallelism="replicas x%d" % world, experts=args.experts),
    }
    line.update(roofline_fields(r, fp8))
    line.update({
        "step_ms_percentiles": {"p10": r["step_pct"][10], "p50": r["step_pct"][50], "p90": r["step_pct"][90]},
        "e2e": {"value": e2e_tokens_per_s, "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"],
                "copies": "every step's x in and y + loss out, on their own streams, overlapping the "
                          "neighbouring steps' layers (double-buffered device buffers)"},
        "gpu_launches": launches_per_forward(wl, fp8) * args.steps,
        "clocks": r["clocks"],
    })
    if "cpu" in r:
        line["cpu_baseline"] = r["cpu"]
    if subs:
        line["sub_records"] = subs
    print(json.dumps(line), flush=True)


def roofline_fields(r, fp8):
    """tflops, layer_roofline, roofline (grouped FFN), stages and routing of
    one measured workload, fractions against the tensor peak its own clock
    record calls for (tensor_peak), burst and sustained fractions beside."""
    peaks = r["peaks"]
    tag = "of measured" if r["peak_src"] == "measured" else "of fallback"
    kind = "fp8 (2 x the measured bf16 figure, the nominal fp8 : bf16 ratio)" if fp8 else "bf16"
    return {
        "tflops": r["flops"] / (r["ms"] * 1e-3) / 1e12,
        "layer_roofline": {"bound": r["bound"], "time_ms": r["layer_roof_ms"],
                           "frac": r["layer_roof_ms"] / r["ms"], "flops": r["flops"],
                           "alg_bytes": r["alg_bytes"],
                           "frac_burst": r["layer_roof_burst_ms"] / r["ms"],
                           "frac_sustained": r["layer_roof_sust_ms"] / r["ms"],
                           "peak_note": "%s %s peak and copy bandwidth, %s" % (r["peak_which"], kind, tag)},
        "roofline": {"kernel": ("grouped_ffn_fp8 (tcgen05 e4m3 gemm1 + H quantization + gemm2)" if fp8
                                else "grouped_ffn (tcgen05 gemm1 + gemm2)"), "bound": "tensor",
                     "achieved": r["ffn_tflops"], "peak": r["peak_t"], "unit": "TFLOP/s",
                     "frac": r["ffn_tflops"] / r["peak_t"], "traffic": r["traffic"],
                     "frac_burst": r["ffn_tflops"] / peaks["bf16_tflops"],
                     "frac_sustained": r["ffn_tflops"] / peaks["bf16_tflops_sustained"],
                     "peak_note": "%s %s peak, %s" % (r["peak_which"], kind, tag)},
        "stages_ms": {k: round(v, 4) for k, v in r["stage_avg"].items()},
        "routing": {"kept_rows": r["kept_rows"], "dropped": r["n_dropped"], "loss": r["loss"],
                    "max_count": int(r["counts"].max()), "min_count": int(r["counts"].min()),
                    "active_experts": int((r["counts"] > 0).sum())},
    }


def backward_record(args, wl, dev, world):
    """The backward pass (moe_backward) after one forward pass: K timed steps,
    L2 flushed between them.  Algorithmic FLOPs: the expert contractions'
    input and weight gradients (2 x the forward's expert FLOPs) plus the
    router's two gradient contractions (2 x 2 T d E); the pre-activation
    recompute the implementation adds is not counted.  Then K training steps
    (moe_forward_train + moe_backward, the forward handing its expert
    pre-activations to the backward), timed per half."""
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    inp = syn.generate(wl, dev, seed=0)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, dev, want_logits=True)
    ws = nat.alloc_workspace(cfg, dev)
    nat.forward(cfg, inp, out, ws, stream)
    g = torch.Generator(device=dev).manual_seed(1)
    dy = torch.randn((wl.T, wl.d_model), generator=g, device=dev).to(torch.bfloat16)
    bws = torch.empty(nat.backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        flush.zero_()
        nat.backward(cfg, inp, out, ws, dy, 0.01, ws=bws, stream=stream)
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(ws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the backward warm-up")
    sampler = ClockSampler(dev.index)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.sub_steps)]
    for i in range(args.sub_steps):
        flush.zero_()
        ev[i][0].record(stream)
        nat.backward(cfg, inp, out, ws, dy, 0.01, ws=bws, stream=stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.sub_steps
    ms = max_over_ranks([ms], world, dev)[0]
    counts = out.counts.cpu().numpy()
    cap = nat.capacity(cfg)
    kept = np.minimum(counts, cap) if cap >= 0 else counts
    flops = 2.0 * wl.expert_flops(int(kept.sum())) + 4.0 * wl.T * wl.d_model * wl.E
    peaks, peak_src = load_peaks()
    peak_t, which = tensor_peak(peaks, clocks)
    tf = flops / (ms * 1e-3) / 1e12

    # a training step: moe_forward_train (the forward that also leaves the
    # expert pre-activations in the backward workspace) and moe_backward
    def train_step(evs):
        evs[0].record(stream)
        nat.forward_train(cfg, inp, out, ws, bws, stream)
        evs[1].record(stream)
        nat.backward(cfg, inp, out, ws, dy, 0.01, ws=bws, stream=stream)
        evs[2].record(stream)

    ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.sub_steps)]
    for _ in range(3):
        flush.zero_()
        train_step(ev3[0])
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(ws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the training-step warm-up")
    for i in range(args.sub_steps):
        flush.zero_()
        train_step(ev3[i])
    torch.cuda.synchronize(dev)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev3) / args.sub_steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev3) / args.sub_steps
    fwd_ms, bwd_ms = max_over_ranks([fwd_ms, bwd_ms], world, dev)
    return {"workload": wl.name, "pass": "backward (dx, dW_r, d logit offset, all expert weight gradients)",
            "steps": args.sub_steps, "warmup": 3, "ms_per_step": ms,
            "tokens_per_s": job_tokens_per_s(world, wl.T, ms), "tflops": tf,
            "training_step": {"entry": "moe_forward_train + moe_backward (pre-activations handed over, no recompute)",
                              "ms_per_step": fwd_ms + bwd_ms, "forward_ms": fwd_ms, "backward_ms": bwd_ms,
                              "backward_tflops": flops / (bwd_ms * 1e-3) / 1e12,
                              "backward_frac": flops / (bwd_ms * 1e-3) / 1e12 / peak_t},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_t, "unit": "TFLOP/s", "frac": tf / peak_t,
                         "flops": flops, "peak_note": "%s bf16 peak, %s" % (which, "of measured" if peak_src ==
                                                                             "measured" else "of fallback")},
            "clocks": clocks}


def mx_record(args, wl, dev, world):
    """The grouped FFN with block-scaled (MX) e4m3 experts (moe_grouped_ffn_mx:
    GEMM 1, the MX quantization of H, GEMM 2) on the workload's routed rows:
    routing, permutation and the MX codes and scale rows of the packed rows
    are produced once before the timed region; K timed steps, L2 flushed
    between them.  Roofline: the expert FLOPs of the kept rows against the
    e4m3 tensor peak (2 x the measured bf16 figure)."""
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    inp = syn.generate(wl, dev, seed=0, weights=False)
    cfg = nat.config_from_workload(wl)
    T, k, E, d = wl.T, wl.top_k, wl.E, wl.d_model
    sld = nat.mx_sld(cfg)
    w = syn.generate_mx_experts(wl, sld, dev, seed=0)
    ws = nat.alloc_workspace(cfg, dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    psum = torch.empty((nat.router_blocks(cfg), E), dtype=torch.float32, device=dev)
    nat.moe_router_topk(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"], idx, gate, None, psum, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    row_token = torch.zeros(T * k, dtype=torch.int32, device=dev)
    row_gate = torch.zeros(T * k, dtype=torch.float32, device=dev)
    nat.moe_permute(cfg, inp["x"], idx, gate, counts, kept, offsets, row_of, row_token, row_gate, None, None, ws)
    x8 = torch.empty((T, d), dtype=torch.uint8, device=dev)
    xs = torch.zeros((T, sld), dtype=torch.uint8, device=dev)
    nat.moe_quantize_rows_mx(inp["x"], x8, xs)
    torch.cuda.synchronize(dev)
    n = int(offsets[-1].item())
    rt = row_token[:n].long()
    x8p = torch.zeros((T * k, d), dtype=torch.uint8, device=dev)
    x8p[:n] = x8[rt]
    xsp = torch.zeros((T * k, sld), dtype=torch.uint8, device=dev)
    xsp[:n] = xs[rt]
    y_perm = torch.empty((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    mws = torch.zeros(nat.grouped_ffn_mx_workspace_size(cfg, sld), dtype=torch.uint8, device=dev)

    def step():
        nat.moe_grouped_ffn_mx(cfg, x8p, xsp, offsets, row_gate, w, sld, w.get("b1"), w.get("b2"), x8, xs, y_perm,
                               mws, stream)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(mws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the MX warm-up")
    sampler = ClockSampler(dev.index)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.sub_steps)]
    for i in range(args.sub_steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.sub_steps
    ms = max_over_ranks([ms], world, dev)[0]
    flops = float(wl.expert_flops(n))
    peaks, peak_src = load_peaks()
    peak_t, which = tensor_peak(peaks, clocks)
    peak_t *= 2.0
    tf = flops / (ms * 1e-3) / 1e12

    # the whole layer with MX experts (moe_forward_mx), timed the same way
    out = nat.Outputs(cfg, dev)
    nat.moe_router_freeze(cfg, inp["Wr"], ws, stream)
    for _ in range(3):
        flush.zero_()
        nat.forward_mx(cfg, inp, w, sld, out, ws, mws, stream)
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(ws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the MX layer warm-up")
    for i in range(args.sub_steps):
        flush.zero_()
        ev[i][0].record(stream)
        nat.forward_mx(cfg, inp, w, sld, out, ws, mws, stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    layer_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in ev) / args.sub_steps], world, dev)[0]
    return {"workload": wl.name, "experts": "mx_e4m3 (32-value E8M0 blocks, tcgen05 block-scaled MMA)",
            "pass": "grouped FFN stage (GEMM 1, H quantization, GEMM 2) on the packed rows",
            "steps": args.sub_steps, "warmup": 3, "ms_per_step": ms, "tflops": tf,
            "layer": {"entry": "moe_forward_mx (router, x quantization, permute, scale-row gather, grouped FFN, "
                               "combine)", "ms_per_step": layer_ms,
                      "tokens_per_s": job_tokens_per_s(world, wl.T, layer_ms),
                      "tflops": flops / (layer_ms * 1e-3) / 1e12},
            "gpu_launches": (4 if wl.d_ff_shared else 3) * args.sub_steps,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_t, "unit": "TFLOP/s", "frac": tf / peak_t,
                         "flops": flops, "peak_note": "e4m3: 2 x the %s bf16 peak (the nominal fp8 : bf16 ratio), %s"
                         % (which, "of measured" if peak_src == "measured" else "of fallback")},
            "clocks": clocks}


def w4_record(args, wl, dev, world):
    """The grouped FFN with INT4 weight-only experts (moe_grouped_ffn_w4: the
    two GEMMs with the weights decoded to bf16 in shared memory each stage)
    on the workload's routed rows, then the whole layer (moe_forward_w4),
    timed like the MX record.  Roofline: the expert FLOPs of the kept rows
    against the bf16 tensor peak, and the packed weight bytes per step."""
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    inp = syn.generate(wl, dev, seed=0, weights=False)
    cfg = nat.config_from_workload(wl)
    T, k, E, d = wl.T, wl.top_k, wl.E, wl.d_model
    sld = nat.w4_sld(cfg)
    w = syn.generate_w4_experts(wl, sld, dev, seed=0)
    ws = nat.alloc_workspace(cfg, dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    psum = torch.empty((nat.router_blocks(cfg), E), dtype=torch.float32, device=dev)
    nat.moe_router_topk(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"], idx, gate, None, psum, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    row_token = torch.zeros(T * k, dtype=torch.int32, device=dev)
    row_gate = torch.zeros(T * k, dtype=torch.float32, device=dev)
    x_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    nat.moe_permute(cfg, inp["x"], idx, gate, counts, kept, offsets, row_of, row_token, row_gate, x_perm, None, ws)
    torch.cuda.synchronize(dev)
    n = int(offsets[-1].item())
    y_perm = torch.empty((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)

    def step():
        nat.moe_grouped_ffn_w4(cfg, x_perm, offsets, row_gate, w, sld, w.get("b1"), w.get("b2"), inp["x"], y_perm,
                               ws, stream)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(ws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the INT4 warm-up")
    sampler = ClockSampler(dev.index)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.sub_steps)]
    for i in range(args.sub_steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.sub_steps
    ms = max_over_ranks([ms], world, dev)[0]
    flops = float(wl.expert_flops(n))
    peaks, peak_src = load_peaks()
    peak_t, which = tensor_peak(peaks, clocks)
    tf = flops / (ms * 1e-3) / 1e12
    wbytes = sum(int(v.numel()) for key, v in w.items() if v is not None and key[0] == "W")

    out = nat.Outputs(cfg, dev)
    nat.moe_router_freeze(cfg, inp["Wr"], ws, stream)
    for _ in range(3):
        flush.zero_()
        nat.forward_w4(cfg, inp, w, sld, out, ws, stream)
    torch.cuda.synchronize(dev)
    if nat.moe_get_device_status(ws, stream) != nat.MOE_OK:
        raise RuntimeError("device status after the INT4 layer warm-up")
    for i in range(args.sub_steps):
        flush.zero_()
        ev[i][0].record(stream)
        nat.forward_w4(cfg, inp, w, sld, out, ws, stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    layer_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in ev) / args.sub_steps], world, dev)[0]
    return {"workload": wl.name, "experts": "int4 weight-only (bf16 scale per 128 inputs, decoded to bf16 in "
                                            "shared memory, tcgen05 kind::f16)",
            "pass": "grouped FFN stage (GEMM 1, GEMM 2) on the packed rows",
            "steps": args.sub_steps, "warmup": 3, "ms_per_step": ms, "tflops": tf,
            "weight_bytes": wbytes,
            "layer": {"entry": "moe_forward_w4 (router, permute, grouped FFN, combine)", "ms_per_step": layer_ms,
                      "tokens_per_s": job_tokens_per_s(world, wl.T, layer_ms),
                      "tflops": flops / (layer_ms * 1e-3) / 1e12},
            "gpu_launches": 2 * args.sub_steps,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_t, "unit": "TFLOP/s", "frac": tf / peak_t,
                         "flops": flops, "peak_note": "bf16 (the MMA's operand type), %s %s"
                         % (which, "of measured" if peak_src == "measured" else "of fallback")},
            "clocks": clocks}


def sub_record(args, spec, dev, world, rank):
    """One further workload timed like the headline one (device-resident steps
    with the L2 flushed between them, the staged per-stage pass), reported
    with its own roofline fractions.  spec: "workload", "workload:fp8",
    "workload:backward" (the backward pass, backward_record), "workload:mx"
    (the MX grouped FFN stage, mx_record) or "workload:w4" (the INT4
    weight-only grouped FFN stage, w4_record)."""
    name, _, experts = spec.partition(":")
    wl = syn.WORKLOADS[name]
    if experts == "backward":
        return backward_record(args, wl, dev, world)
    if experts == "mx":
        return mx_record(args, wl, dev, world)
    if experts == "w4":
        return w4_record(args, wl, dev, world)
    fp8 = experts == "fp8"
    r = run_ours(args, wl, dev, world, rank, fp8=fp8, steps=args.sub_steps, warmup=3, full=False)
    rec = {"workload": name, "experts": "fp8" if fp8 else "bf16", "steps": args.sub_steps, "warmup": 3,
           "ms_per_step": r["ms"], "tokens_per_s": job_tokens_per_s(world, wl.T, r["ms"]),
           "step_ms_percentiles": {"p10": r["step_pct"][10], "p50": r["step_pct"][50], "p90": r["step_pct"][90]},
           "gpu_launches": launches_per_forward(wl, fp8) * args.sub_steps, "clocks": r["clocks"]}
    rec.update(roofline_fields(r, fp8))
    return rec


if __name__ == "__main__":
    main()
