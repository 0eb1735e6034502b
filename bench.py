#!/usr/bin/env python
"""Decode throughput of the expert-cache MoE path on B200.

Workload (one "step" = one batch-1 decode token through the whole hot path): a 40-layer
pre-norm MoE stack, hidden 2048, 256 experts, top-8, SwiGLU 512 plus a 512-wide shared
expert, GGUF Q4_0 expert weights, Zipf(1.0)-biased router over seeded per-layer
permutations, tokens x ~ N(0, 1).  Timed at 100% expert residency (the value) and at
60% residency with the hot set pinned from a calibration histogram (2048 tokens of a
separate stream, the length of the prefill prompt; --calib-steps) plus an
8-slot LRU ring per layer, cold experts in pinned host memory (Luce Spark write-up,
theneuralfeed.com, key components), and with a uniform 60% placement for contrast.

Prints one JSON line (rank 0).  --impl reference times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "MoE decode tok/s at 100%/60% expert residency; fraction of HBM/PCIe roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TFLOPS = 1400.0  # sustained dense bf16, an earlier measurement on this machine
# DRAM bytes (read + write) of one 40-layer decode launch, from the ncu capture of the
# 4-layer case scaled by 10, valid only for the kernel source it was taken on; any other
# source reports null.
TRAFFIC_REF = {"kernel_sha256_prefix": "c2b549be9b6e7e69", "bytes_per_launch": 689.78176e6}
WORKLOAD = ("40-layer MoE decode stack, hidden 2048, 256 experts top-8, SwiGLU 512 + shared 512, "
            "Q4_0, Zipf router; batch-1 tokens; 100% residency (value) and 60% calibrated "
            "residency + 8-slot LRU ring (residency_60)")


def compact(obj, digits=5):
    """Floats rounded to `digits` significant digits, recursively (keeps the JSON line short)."""
    if isinstance(obj, float):
        return float(f"{obj:.{digits}g}")
    if isinstance(obj, dict):
        return {k: compact(v, digits) for k, v in obj.items()}
    if isinstance(obj, (list, tuple)):
        return [compact(v, digits) for v in obj]
    return obj


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def traffic_per_launch(n_layers: int):
    import hashlib
    src = os.path.join(ROOT, "expert_cache_host_router_b200", "csrc", "decode_kernel.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if sha != TRAFFIC_REF["kernel_sha256_prefix"] or n_layers != 40:
        return None
    return TRAFFIC_REF["bytes_per_launch"]


def active_bytes_per_token(s) -> int:
    """Algorithmic expert bytes of one token: L * (k + shared) experts' Q4_0 weights."""
    per = 3 * s.hidden * s.inter * 18 // 32
    sh = 3 * s.hidden * s.shared_inter * 18 // 32
    return s.n_layers * (s.top_k * per + sh)


class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) while the GPU is busy."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def reduce_over_ranks(value_ms: float, units: float, world: int):
    """Max of the per-rank times and sum of the per-rank units (replicas)."""
    if world == 1:
        return value_ms, units
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ------------------------------------------------------------------ CPU oracle legs

def oracle_tokens_per_s(shape, n_layers: int, n_tokens: int, warmup: int = 0, layers=None):
    """The oracle, as it stands, on n_tokens tokens through the first n_layers layers;
    returns (tok/s scaled to the full stack, seconds, threads)."""
    import oracle
    sub = synthetic.Shape(n_layers, shape.hidden, shape.n_experts, shape.top_k, shape.inter,
                          shape.shared_inter, shape.ring_slots, shape.use_rmsnorm, shape.zipf_s)
    if layers is None:
        layers = [synthetic.layer_weights(l, shape) for l in range(n_layers)]
    layers = layers[:n_layers]
    m = oracle.Model(sub, layers)
    for i in range(warmup):
        m.decode(synthetic.token(i, shape.hidden))
    t0 = time.perf_counter()
    for i in range(n_tokens):
        m.decode(synthetic.token(warmup + i, shape.hidden))
    dt = time.perf_counter() - t0
    return n_tokens * n_layers / shape.n_layers / dt, dt, 1


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    shape = synthetic.FULL_STACK
    sample_layers = 4
    tps, dt, cores = oracle_tokens_per_s(shape, sample_layers, args.steps, args.warmup)
    sample = (f"{args.steps} timed steps (after {args.warmup} warm-up), each one token through "
              f"{sample_layers} of the 40 layers, scaled to full tokens")
    line = {"impl": "reference", "metric": METRIC, "value": tps, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "layers": 40},
            "cpu_baseline": {"value": tps, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tps, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_drift(args, shape, layers, local, dev, xs_steps=1024, switch=512, every=64,
              fraction=0.4, ring=4):
    """Online recalibration under drift: the stack at 40% residency with 4-slot rings;
    the router bias (traffic popularity) switches to reshuffled Zipf permutations at
    token 512 of 1024; cold-hit rates before / after the switch for calibrated placement
    with recalibration every 64 tokens, calibrated placement frozen, and uniform."""
    import dataclasses

    import torch

    import expert_cache_host_router_b200 as moe
    s = dataclasses.replace(shape, ring_slots=ring)
    m = moe.ExpertCacheMoE(s, device=local, log_steps=xs_steps + 256)
    for l in range(s.n_layers):
        m.load_layer(l, layers[l])
    new_bias = [synthetic.zipf_bias(l, s.n_experts, s.zipf_s, synthetic.SEED_RESHUFFLE)
                for l in range(s.n_layers)]
    n_cal = args.drift_calib_steps
    calib = torch.from_numpy(synthetic.tokens(0, n_cal, s.hidden, synthetic.SEED_CALIB)).to(dev)
    xs = torch.from_numpy(synthetic.tokens(0, xs_steps, s.hidden)).to(dev)
    y = torch.empty(s.hidden, dtype=torch.float32, device=dev)
    m.set_residency(1.0)
    for i in range(n_cal):
        m.decode(calib[i], y)
    m.sync()
    _, hist, _ = m.stats(reset=True, log_cap=n_cal * s.n_layers * s.top_k)
    out = {"residency": fraction, "ring_slots": ring, "steps": xs_steps, "reshuffle_at": switch,
           "recalibrate_every": every, "calibration_tokens": n_cal}
    stream = torch.cuda.current_stream(dev)
    for name, place, recal in (("calibrated_recal", moe.MOE_PLACE_CALIBRATED, True),
                               ("calibrated_static", moe.MOE_PLACE_CALIBRATED, False),
                               ("uniform", moe.MOE_PLACE_UNIFORM, False)):
        for l in range(s.n_layers):
            m.set_router_bias(l, layers[l].bias)
        m.set_residency(fraction, hist, place)
        m.stats(reset=True, log_cap=(xs_steps + 256) * s.n_layers * s.top_k)
        ms = [0.0, 0.0]
        for half, (a, b) in enumerate(((0, switch), (switch, xs_steps))):
            if half == 1:
                for l in range(s.n_layers):
                    m.set_router_bias(l, new_bias[l])
            t_dev = 0.0
            for t0 in range(a, b, every):
                if recal and t0:
                    m.recalibrate()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for t in range(t0, min(b, t0 + every)):
                    m.decode(xs[t], y)
                e1.record(stream)
                m.sync()
                t_dev += e0.elapsed_time(e1)
            ms[half] = t_dev
        st, _, log = m.stats(log_cap=xs_steps * s.n_layers * s.top_k)
        kinds = log["kind"].reshape(xs_steps, -1)
        res = {}
        for half, (a, b) in enumerate(((0, switch), (switch, xs_steps))):
            k = kinds[a:b]
            res["before" if half == 0 else "after"] = {
                "cold_hit_rate": float(np.mean(k != moe.MOE_PIN_HIT)),
                "misses_per_token": float(np.sum(k == moe.MOE_MISS)) / (b - a),
                "tok_s": (b - a) / (ms[half] * 1e-3)}
        res["repins"] = st["repins"]
        res["repin_copies"] = st["repin_copies"]
        out[name] = res
    m.close()
    return out


def decode_point(m, shape, xs, y, stream, steps):
    """Decode `steps` tokens of xs on m as placed now: tok/s (CUDA events), cold-hit rate
    and miss copies per token from the run's own log."""
    import torch
    m.stats(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        m.decode(xs[i], y)
    e1.record(stream)
    m.sync()
    st, _, _ = m.stats(reset=True)
    acc = max(st["accesses"], 1)
    return {"tok_s": steps / (e0.elapsed_time(e1) * 1e-3),
            "cold_hit_rate": (st["ring_hits"] + st["misses"]) / acc,
            "misses_per_token": st["misses"] / steps}


def run_residency_curve(m, shape, hist, xs, y, stream, steps=128):
    """tok/s and cold-hit rate over residency 1.0, 0.8, 0.6, 0.4 for calibrated placement
    (pinned = top-P of the calibration histogram) and uniform placement (experts 0..P-1):
    the offload comparison the write-up makes at one point, as a curve."""
    import expert_cache_host_router_b200 as moe
    out = []
    for rho in (1.0, 0.8, 0.6, 0.4):
        for name, place in (("calibrated", moe.MOE_PLACE_CALIBRATED), ("uniform", moe.MOE_PLACE_UNIFORM)):
            if rho == 1.0 and place == moe.MOE_PLACE_UNIFORM:
                continue  # every expert pinned: the same placement
            m.set_residency(rho, hist, place)
            out.append({"residency": rho, "placement": name, **decode_point(m, shape, xs, y, stream, steps)})
    return out


def run_small_stack(dev, local, calib_steps, steps=256, warmup=8):
    """The 40-layer stack at the small layer shape (hidden 512, 64 experts, top-4, SwiGLU
    256, no shared expert) at 100% and at 60% residency (calibrated and uniform), 8-slot
    rings."""
    import dataclasses

    import torch

    import expert_cache_host_router_b200 as moe
    s = dataclasses.replace(synthetic.SMALL, n_layers=40, use_rmsnorm=1, ring_slots=8, zipf_s=1.0)
    m = moe.ExpertCacheMoE(s, device=local, log_steps=max(4096, steps + warmup + 16))
    for l in range(s.n_layers):
        m.load_layer(l, synthetic.layer_weights(l, s))
    y = torch.empty(s.hidden, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    m.set_residency(1.0)
    calib = torch.from_numpy(synthetic.tokens(0, calib_steps, s.hidden, synthetic.SEED_CALIB)).to(dev)
    for i in range(calib_steps):
        m.decode(calib[i], y)
    m.sync()
    _, hist, _ = m.stats(reset=True)
    xs = torch.from_numpy(synthetic.tokens(0, warmup + steps, s.hidden)).to(dev)
    out = {"shape": {"layers": 40, "hidden": 512, "experts": 64, "top_k": 4, "inter": 256, "shared_inter": 0,
                     "ring_slots": 8},
           "active_bytes_per_token": active_bytes_per_token(s)}
    for name, rho, place in (("100", 1.0, moe.MOE_PLACE_CALIBRATED), ("60_calibrated", 0.6, moe.MOE_PLACE_CALIBRATED),
                             ("60_uniform", 0.6, moe.MOE_PLACE_UNIFORM)):
        m.set_residency(rho, hist, place)
        for i in range(warmup):
            m.decode(xs[i], y)
        m.sync()
        out[name] = decode_point(m, s, xs[warmup:], y, stream, steps)
    m.close()
    return out


def run_prefill(m, shape, dev, n_tokens=2048, warmup=2, runs=5):
    """Batched prefill of n_tokens through the whole stack at full residency (tcgen05
    grouped GEMM path), timed with CUDA events on the launching stream.  Roofline: per
    layer and expert, max(its FLOPs at the measured dense tensor peak, its weight bytes
    at the measured HBM bandwidth), summed; token counts per expert from the routing
    histogram of the timed runs."""
    import torch
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    tflops = float(peaks.get("bf16_tflops_sustained", FALLBACK_TFLOPS))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    x = torch.from_numpy(synthetic.tokens(50000, n_tokens, shape.hidden)).to(dev)
    y = torch.empty_like(x)
    m.set_residency(1.0)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        m.prefill(x, y)
    m.sync()
    m.stats(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(runs):
        m.prefill(x, y)
    e1.record(stream)
    m.sync()
    ms = e0.elapsed_time(e1) / runs
    _, hist, _ = m.stats(reset=True)
    n_e = hist.astype(np.float64) / runs  # [L][E] tokens per expert per pass
    roof = prefill_roofline(n_e, n_tokens, shape, tflops, hbm)
    sec = ms * 1e-3
    return {"tokens": n_tokens, "value": n_tokens / sec, "unit": "tok/s", "ms": ms, "runs": runs,
            "dtype": "q4_0 -> fp16 weights x fp16 hi+lo activations, fp32 accumulate (tcgen05)",
            "roofline": {"bound": "tensor", "achieved": roof["useful_flops"] / sec / 1e12, "peak": tflops,
                         "unit": "TFLOP/s", "frac": roof["time_s"] / sec, "roofline_ms": roof["time_s"] * 1e3,
                         "peak_kind": "measured sustained bf16 (fp16 same rate)",
                         "issued_tflops": roof["issued_flops"] / sec / 1e12,
                         "note": "frac = per-expert max(flop, weight-byte) time summed / measured time"}}


def prefill_roofline(n_e, n_tokens, shape, tflops, hbm_gbs):
    """Roofline of a prefill pass: per layer and routed expert, the larger of its FLOPs at
    the tensor peak and its Q4_0 weight bytes at HBM bandwidth (experts no token chose
    cost nothing), plus the shared expert (every token) per layer.  n_e: [L][E] tokens per
    expert.  Also the useful FLOPs and the FLOPs the kernels issue (128-row tiles, each
    K step twice: activation hi and lo)."""
    n_e = np.asarray(n_e, np.float64)
    H, I, Is = shape.hidden, shape.inter, shape.shared_inter
    fl_tok = 2.0 * 3 * H * I  # one token through one routed expert
    by_exp = 3 * H * I * 18 / 32
    t = float(np.sum(np.maximum(n_e * fl_tok / (tflops * 1e12), np.where(n_e > 0, by_exp, 0.0) / (hbm_gbs * 1e9))))
    if Is > 0:
        t += shape.n_layers * max(n_tokens * 2.0 * 3 * H * Is / (tflops * 1e12), 3 * H * Is * 18 / 32 / (hbm_gbs * 1e9))
    useful = float(np.sum(n_e) * fl_tok + shape.n_layers * n_tokens * 2.0 * 3 * H * Is)
    issued = float(np.sum(np.ceil(n_e / 128.0))) * 128 * 2.0 * 3 * H * I * 2
    if Is > 0:
        issued += shape.n_layers * np.ceil(n_tokens / 128.0) * 128 * 2.0 * 3 * H * Is * 2
    return {"time_s": t, "useful_flops": useful, "issued_flops": float(issued)}


def decode_precision(m, shape, layers, dev):
    """Largest per-layer error of one traced decode token (full residency) against the
    oracle run on the GPU's own layer input, as a fraction of the 2e-3 x RMS bar."""
    import torch

    import oracle
    orc = oracle.Model(shape, layers)
    ht = torch.zeros((shape.n_layers + 1, shape.hidden), dtype=torch.float32, device=dev)
    m.set_trace(ht, None)
    m.decode(torch.from_numpy(synthetic.token(900, shape.hidden)).to(dev))
    m.sync()
    m.set_trace(None, None)
    h = ht.cpu().numpy()
    worst = 0.0
    for l in range(shape.n_layers):
        ref = orc.layer(l, h[l])
        rms = float(np.sqrt(np.mean(ref["y"] ** 2)))
        err = float(np.max(np.abs(h[l + 1].astype(np.float64) - ref["h_out"])))
        worst = max(worst, err / (2e-3 * rms))
    # prefill: 16 tokens through the whole stack, two of them checked at every layer
    T = 16
    hp = torch.zeros((shape.n_layers + 1, T, shape.hidden), dtype=torch.float32, device=dev)
    sp = torch.zeros((shape.n_layers, T, shape.top_k), dtype=torch.int32, device=dev)
    m.set_prefill_trace(hp, sp)
    m.prefill(torch.from_numpy(synthetic.tokens(901, T, shape.hidden)).to(dev))
    m.sync()
    m.set_prefill_trace(None, None)
    hpn = hp.cpu().numpy()
    worst_p = 0.0
    for t in (0, T - 1):
        for l in range(shape.n_layers):
            ref = orc.layer(l, hpn[l, t])
            rms = float(np.sqrt(np.mean(ref["y"] ** 2)))
            err = float(np.max(np.abs(hpn[l + 1, t].astype(np.float64) - ref["h_out"])))
            worst_p = max(worst_p, err / (2e-3 * rms))
    return {"decode_max_layer_err_over_bar": round(worst, 4),
            "prefill_max_layer_err_over_bar": round(worst_p, 4), "bar": "2e-3 x RMS(y) per element",
            "sample": "decode: one token, prefill: two of 16 tokens; every layer, teacher-forced"}


def write_phase_table(m, shape, xs, y, path, n_tokens=8, residency=1.0, hist=None):
    """Per-layer phase times of CTA 0 (median over n_tokens tokens at the given residency)
    from the kernel's marks, plus every CTA's skew, written as JSON to path."""
    import torch

    import expert_cache_host_router_b200 as moe
    n_sm = torch.cuda.get_device_properties(y.device).multi_processor_count
    words = moe.phase_trace_words(shape.n_layers, n_sm)
    st = torch.zeros(words, dtype=torch.int64, device=y.device)
    m.set_residency(residency, hist)
    m.set_phase_trace(st)
    runs = []
    for i in range(n_tokens):
        m.decode(xs[i % len(xs)], y)
        m.sync()
        runs.append(st.cpu().numpy().copy())
    m.set_phase_trace(None)
    L = shape.n_layers
    marks = np.stack([r[: (L + 1) * 32].reshape(L + 1, 32) for r in runs]).astype(np.float64)
    # CTA 0's marks are SM cycles; the kernel's start and end on both clocks give ns per cycle
    ns_per_cycle = float(np.median((marks[:, L, 5] - marks[:, L, 4]) / (marks[:, L, 2] - marks[:, L, 0])))
    names = {1: "prev_layer_output", 2: "h_updated", 10: "norm_u", 11: "own_logit", 12: "x_quantised",
             3: "logits_published", 4: "logits_read", 13: "topk", 14: "cache", 5: "routed", 15: "loads_issued_t0",
             6: "loads_issued", 7: "gateup_done", 16: "swiglu", 17: "down_landed", 18: "down_adds", 19: "fence",
             8: "units_done", 9: "arrived"}
    table = []
    for l in range(L):
        row = {"layer": l}
        for k, n in names.items():
            row[n] = float(np.median(marks[:, l, k] - marks[:, l, 0])) * ns_per_cycle / 1e3
        nxt = marks[:, l + 1, 0] if l + 1 < L else marks[:, L, 2]
        row["layer_us"] = float(np.median(nxt - marks[:, l, 0])) * ns_per_cycle / 1e3
        table.append(row)
    total = float(np.median(marks[:, L, 5] - marks[:, L, 4])) / 1e3
    raw = [float(np.median(marks[:, 1:L, k] - marks[:, 1:L, 0])) * ns_per_cycle / 1e3 for k in range(32)]
    # every CTA's global-timer marks: [0] routing decided, [1] units done, [2] arrival posted,
    # [3] own logits published
    cta = np.stack([r[(L + 1) * 32:].reshape(L, n_sm, 4) for r in runs]).astype(np.float64)  # [tok][L][cta][4]
    rt, ud, ar = cta[..., 0], cta[..., 1], cta[..., 2]
    work = ud - rt  # per CTA: routing decided -> its units done
    cta_stats = {"routed_spread_us": float(np.median(rt.max(axis=2) - rt.min(axis=2))) / 1e3,
                 "units_median_us": float(np.median(np.median(work, axis=2))) / 1e3,
                 "units_max_us": float(np.median(work.max(axis=2))) / 1e3,
                 "arrival_spread_us": float(np.median(ar.max(axis=2) - ar.min(axis=2))) / 1e3,
                 "last_arrival_after_first_routed_us": float(np.median(ar.max(axis=2) - rt.min(axis=2))) / 1e3,
                 "publish_spread_us": float(np.median(cta[..., 3].max(axis=2) - cta[..., 3].min(axis=2))) / 1e3,
                 "last_publishers": [int(c) for c in np.argsort(-np.bincount(
                     cta[..., 3].argmax(axis=2).ravel(), minlength=n_sm))[:6]],
                 "last_to_finish_units": [int(c) for c in np.argsort(-np.bincount(
                     ud.argmax(axis=2).ravel(), minlength=n_sm))[:6]],
                 "slowest_units": [int(c) for c in np.argsort(-np.median(work, axis=(0, 1)))[:6]],
                 # per CTA, median over tokens and layers: how long after the first CTA it
                 # published its logits / posted its arrival
                 "publish_late_us": [round(float(v) / 1e3, 3) for v in np.median(
                     cta[..., 3] - cta[..., 3].min(axis=2, keepdims=True), axis=(0, 1))],
                 "arrival_late_us": [round(float(v) / 1e3, 3) for v in np.median(
                     ar - ar.min(axis=2, keepdims=True), axis=(0, 1))]}
    with open(path, "w") as f:
        json.dump({"unit": "us since layer start (CTA 0), median over tokens", "tokens": n_tokens,
                   "ns_per_cycle": ns_per_cycle, "raw_slots_us": raw, "cta_stats": cta_stats,
                   "kernel_us": total, "layers": table}, f, indent=1)


# ------------------------------------------------------------------ GPU arm

def run_ours(args):
    import torch

    import expert_cache_host_router_b200 as moe
    from expert_cache_host_router_b200 import build as libbuild

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        libbuild.build()
    if world > 1:
        dist.barrier()
    shape = synthetic.FULL_STACK
    if args.layers != shape.n_layers:  # a shorter stack of the same layers (profiling cases)
        import dataclasses
        shape = dataclasses.replace(shape, n_layers=args.layers)
    dev = torch.device("cuda", local)
    keep_layers = rank == 0 and world == 1 and not args.no_cpu_baseline and args.layers == 40
    t0 = time.time()
    layers = [synthetic.layer_weights(l, shape) for l in range(shape.n_layers)]
    gen_s = time.time() - t0
    m = moe.ExpertCacheMoE(shape, device=local, log_steps=max(4096, args.steps + args.warmup + 16))
    if any(args.prefetch):
        m.set_prefetch(*args.prefetch)
    t0 = time.time()
    for l in range(shape.n_layers):
        m.load_layer(l, layers[l])
    load_s = time.time() - t0

    if args.only_prefill:  # the batched-prefill measurement alone (profiling runs)
        line = {"metric": "prefill tok/s", "config": {"workload": f"batched prefill, {shape.n_layers}-layer stack"},
                "prefill": run_prefill(m, shape, dev, runs=args.prefill_runs)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        m.close()
        return
    stream = torch.cuda.current_stream(dev)
    n_tok = args.warmup + args.steps
    xs = torch.from_numpy(synthetic.tokens(0, n_tok, shape.hidden)).to(dev)
    y = torch.empty(shape.hidden, dtype=torch.float32, device=dev)

    # calibration histogram: --calib-steps tokens of a separate stream at full residency
    m.set_residency(1.0)
    calib = torch.from_numpy(synthetic.tokens(0, args.calib_steps, shape.hidden, synthetic.SEED_CALIB)).to(dev)
    for i in range(args.calib_steps):
        m.decode(calib[i], y)
    m.sync()
    _, hist, _ = m.stats(reset=True)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
            torch.cuda.synchronize()

    def timed():
        for i in range(args.warmup):
            m.decode(xs[i], y)
        m.sync()
        m.stats(reset=True)
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            m.decode(xs[args.warmup + i], y)
            ends[i].record(stream)
        e1.record(stream)
        barrier()
        total = e0.elapsed_time(e1)
        per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        m.sync()
        st, _, _ = m.stats(reset=True)
        return total, per, st

    peak, peak_kind = measured_peaks()
    bytes_tok = active_bytes_per_token(shape)
    slot_bytes = 3 * shape.hidden * shape.inter * 18 // 32

    with ClockSampler(local) as clk:
        m.set_residency(1.0)
        t100, per100, st100 = timed()
        if args.phases == "all":
            m.set_residency(0.6, hist, moe.MOE_PLACE_CALIBRATED)
            t60, per60, st60 = timed()
            m.set_miss_path(moe.MOE_MISS_SM_PULL)
            m.set_residency(0.6, hist, moe.MOE_PLACE_CALIBRATED)
            t60p, per60p, st60p = timed()
            m.set_miss_path(moe.MOE_MISS_COPY_ENGINE)
            m.set_residency(0.6, hist, moe.MOE_PLACE_UNIFORM)
            t60u, per60u, st60u = timed()
        else:  # full residency only: no miss copies (profilers serialise the proxy's copies)
            t60, per60, st60 = t100, per100, st100
            t60p, per60p, st60p = t100, per100, st100
            t60u, per60u, st60u = t100, per100, st100

    # host-to-device rate of the miss path: the library's own copy (pinned host tier ->
    # device slot, cudaMemcpyAsync on the proxy's side stream), back to back
    m.set_residency(1.0)
    h2d_gbs = m.measure_h2d(64)
    # and the copies the proxy made during the 60% run, each timed on the device
    h2d_run = (st60["copies_timed"] * slot_bytes / (st60["copy_ns_timed"] * 1e-9) / 1e9
               if st60.get("copies_timed") else None)

    precision = None
    if args.phases == "all" and keep_layers:
        precision = decode_precision(m, shape, layers, dev)

    # end to end through the host-buffer entry point at full residency
    m.set_residency(1.0)
    xh = synthetic.tokens(0, n_tok, shape.hidden)
    for i in range(args.warmup):
        m.decode_host(xh[i])
    barrier()
    t0 = time.perf_counter()
    for i in range(args.steps):
        m.decode_host(xh[args.warmup + i])
    e2e_s = time.perf_counter() - t0
    e2e_ms, e2e_units = reduce_over_ranks(1e3 * e2e_s, args.steps, world)

    t100_max, units100 = reduce_over_ranks(t100, args.steps, world)
    t60_max, units60 = reduce_over_ranks(t60, args.steps, world)
    t60p_max, units60p = reduce_over_ranks(t60p, args.steps, world)
    value100 = units100 / (t100_max * 1e-3)
    value60 = units60 / (t60_max * 1e-3)
    value60p = units60p / (t60p_max * 1e-3)
    value60u = args.steps * world / (max(t60u, 1e-9) * 1e-3)
    kern_ms = statistics.mean(per100)
    achieved = bytes_tok / (kern_ms * 1e-3) / 1e9

    def cache_summary(st):
        acc = max(st["accesses"], 1)
        return {"cold_hit_rate": round((st["ring_hits"] + st["misses"]) / acc, 5),
                "miss_rate": round(st["misses"] / acc, 5),
                "misses_per_token": round(st["misses"] / args.steps, 4),
                "staged_misses": st["staged_misses"]}

    def roof60(st, t_ms, link_gbs):
        miss_bytes = st["misses"] / args.steps * slot_bytes
        r = max(bytes_tok / (peak * 1e9), miss_bytes / (link_gbs * 1e9))
        return {"roofline_frac": round(r / (t_ms * 1e-3 / args.steps), 4), "roofline_us_per_token": round(r * 1e6, 2)}

    c60 = cache_summary(st60)
    line = {
        "metric": METRIC, "value": value100, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t100_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "q4_0 x int16 codes, int32 dot, fp32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": shape.n_layers, "hidden": shape.hidden,
                   "experts": shape.n_experts, "top_k": shape.top_k, "inter": shape.inter,
                   "shared_inter": shape.shared_inter, "ring_slots": shape.ring_slots,
                   "calibration_tokens": args.calib_steps, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: 637 MB of expert weights streamed per token"},
        "residency_60": {"value": value60, "unit": "tok/s", "ratio_to_100": round(value60 / value100, 4),
                         "miss_path": "copy engine (proxy thread)",
                         **roof60(st60, t60_max, h2d_gbs), "h2d_gbs": round(h2d_gbs, 2),
                         "h2d_gbs_miss_copies": None if h2d_run is None else round(h2d_run, 2),
                         **c60,
                         "sm_pull": {"value": value60p, "ratio_to_100": round(value60p / value100, 4),
                                     **roof60(st60p, t60p_max, h2d_gbs), **cache_summary(st60p)},
                         "uniform_placement": {"value": value60u, **cache_summary(st60u)}},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic_per_launch(shape.n_layers), "peak_kind": peak_kind,
                     "kernel": "moe_decode_kernel", "bytes_per_launch": bytes_tok,
                     "mean_launch_ms": kern_ms},
        "e2e": {"value": e2e_units / (e2e_ms * 1e-3), "unit": "tok/s",
                "h2d_bytes_per_step": 4 * shape.hidden, "d2h_bytes_per_step": 4 * shape.hidden + 4},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "setup": {"generate_s": round(gen_s, 1), "load_s": round(load_s, 1), "phases": args.phases},
    }
    if precision is not None:
        line["precision"] = precision
    if args.phase_trace:
        write_phase_table(m, shape, xs, y, args.phase_trace)
        if args.phases == "all":  # where the misses of the 60% placement stall a layer
            write_phase_table(m, shape, xs, y, args.phase_trace.replace(".json", "_60.json"), n_tokens=32,
                              residency=0.6, hist=hist)
            m.set_residency(1.0)
    if args.prefetch_sweep:
        sweep = []
        m.set_residency(1.0)
        for pre, l2 in ((0, 0), (0, 2), (0, 4), (0, 8), (0, 12), (4, 0), (8, 0), (0, 0)):
            m.set_prefetch(pre, l2)
            for i in range(args.warmup):
                m.decode(xs[i], y)
            sweep.append({"preload": pre, "l2": l2, **decode_point(m, shape, xs[args.warmup:], y, stream,
                                                                 min(64, args.steps))})
        m.set_prefetch(*args.prefetch)
        line["prefetch_sweep"] = sweep
    if args.phases == "all" and not args.no_curve:
        line["residency_curve"] = run_residency_curve(m, shape, hist, xs, y, stream, steps=min(128, len(xs)))
    if args.phases == "all" and not args.no_prefill:
        line["prefill"] = run_prefill(m, shape, dev, runs=args.prefill_runs)
    m.close()
    del m
    if args.phases == "all" and not args.no_drift:
        line["drift"] = run_drift(args, shape, layers, local, dev, xs_steps=1024)
    if args.phases == "all" and not args.no_curve:
        line["small_stack"] = run_small_stack(dev, local, args.calib_steps)
    if keep_layers:
        tps, dt, cores = oracle_tokens_per_s(shape, shape.n_layers, args.cpu_tokens, layers=layers)
        line["cpu_baseline"] = {"value": tps, "unit": "tok/s", "cores": cores, "kind": "oracle",
                                "sample": f"{args.cpu_tokens} tokens through all 40 layers ({dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(compact(line, 6)), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--calib-steps", type=int, default=2048,
                    help="tokens of the calibration stream whose routing histogram picks the pinned set")
    ap.add_argument("--drift-calib-steps", type=int, default=128,
                    help="calibration tokens of the drift run (before its recalibrations take over)")
    ap.add_argument("--cpu-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=40, help="stack depth (40 = the benchmark workload)")
    ap.add_argument("--no-drift", action="store_true", help="skip the recalibration-under-drift run")
    ap.add_argument("--no-prefill", action="store_true", help="skip the batched-prefill run")
    ap.add_argument("--only-prefill", action="store_true", help="run only the batched-prefill measurement")
    ap.add_argument("--no-curve", action="store_true",
                    help="skip the residency curve and the small-shape stack")
    ap.add_argument("--prefill-runs", type=int, default=5, help="timed prefill passes")
    ap.add_argument("--prefetch", type=int, nargs=2, default=[0, 0], metavar=("PRELOAD", "L2"),
                    help="likely experts per layer preloaded into shared memory / prefetched into L2")
    ap.add_argument("--prefetch-sweep", action="store_true", help="decode tok/s at 100%% over prefetch depths")
    ap.add_argument("--phase-trace", default=None, help="write a per-layer phase table (JSON) to this path")
    ap.add_argument("--phases", default="all", choices=["all", "100"],
                    help="'100' times full residency only (no miss copies), for profiler runs")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
