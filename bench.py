#!/usr/bin/env python
"""Canvas denoising step benchmark: canvas tokens/sec on one B200 at fixed
denoise steps, and the fraction of the HBM roofline.

Workload ("stack"): the 30-layer synthetic stack (25 local layers with a
1024-key window over the prompt, 5 global layers), d_model 2816, 16 query / 8
key-value heads of 256, 128 experts top-8 + 1 shared (width 704), tied vocab
262144, a 256-slot canvas, a 4096-token prompt K/V per layer, batch 1, 8
denoising steps per block.  Weights are seeded random (bf16), the prompt K/V
and canvas synthetic.

A step is one full pass (embedding, 30 blocks, vocab head, commit) through
the C ABI.  canvas tok/s = batch * 256 tokens finalised per 8 steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun), every rank runs its own replica on its own
GPU (independent canvases, no collective on the data path; weak scaling); the
timed region is bracketed by barriers and the reported time is the max over
ranks.  --impl reference times the CPU oracle as the reference arm.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "canvas tokens/sec on 1 B200 (fixed denoise steps); % of HBM roofline per step"
sys.path.insert(0, ROOT)

WORKLOAD = "stack"


def workload_desc(cfg):
    skew = f", Zipf({cfg['zipf_s']}) expert popularity" if cfg.get("zipf_s") else ""
    return (f"{cfg['n_layers']}-layer canvas denoising stack: d_model {cfg['d_model']}, "
            f"{cfg['n_q_heads']}q/{cfg['n_kv_heads']}kv heads x {cfg['head_dim']}, "
            f"{cfg['n_experts']} experts top-{cfg['top_k']} + {cfg['n_shared']} shared "
            f"(width {cfg['d_ff']}), vocab {cfg['vocab']} tied, canvas {cfg['canvas_len']}, "
            f"prompt K/V {cfg['prompt_len']} per layer (window {cfg['window']} on 5 of 6 layers), "
            f"batch {cfg['batch']}, {cfg['steps']} steps per block{skew}")


def config_json(cfg, n_gpus):
    extra = {"expert_weights": "fp8 e4m3, one fp32 scale per weight row"} if cfg.get("expert_fp8") \
        else {}
    return {"workload": workload_desc(cfg), "name": cfg["name"], "batch": cfg["batch"], **extra,
            "canvas_len": cfg["canvas_len"], "prompt_len": cfg["prompt_len"],
            "steps_per_block": cfg["steps"], "n_layers": cfg["n_layers"],
            "l2": "inputs larger than L2: ~50 GB of weights streamed from HBM every step",
            "parallelism": "replicas" if n_gpus > 1 else "single"}


# ----------------------------------------------------------------------------- algorithmic bytes

def bytes_per_step(cfg, active_experts=None):
    """Algorithmic HBM bytes of one pass: every weight the pass needs once (the
    dense projections, the router, the shared expert and the routed experts
    that receive rows -- `active_experts` per layer on average, all of them when
    None), each layer's visible prompt K/V once, and the tied embedding once."""
    d, F, E = cfg["d_model"], cfg["d_ff"], cfg["n_experts"]
    dh, Hq, Hkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    P, W, L = cfg["prompt_len"], cfg["window"], cfg["n_layers"]
    act = E if active_experts is None else active_experts
    dense = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d)
    experts = (act + cfg["n_shared"]) * expert_group_bytes(cfg)
    kv = 0
    for l in range(L):
        vis = P if (l + 1) % cfg["global_every"] == 0 else min(W, P)
        kv += 2 * cfg["batch"] * Hkv * vis * dh * 2
    head = cfg["vocab"] * d * 2
    return L * (dense + experts) + kv + head


def expert_group_bytes(cfg, part="all"):
    """Weight bytes of one expert group: bf16, or (expert_fp8) one byte a code plus a
    4-byte scale per weight row.  part: "gateup", "down" or "all"."""
    d, F = cfg["d_model"], cfg["d_ff"]
    if cfg.get("expert_fp8"):
        gu, dn = 2 * F * d + 4 * 2 * F, d * F + 4 * d
    else:
        gu, dn = 2 * 2 * F * d, 2 * d * F
    return {"gateup": gu, "down": dn, "all": gu + dn}[part]


def gateup_bytes_per_launch(cfg, active_experts=None):
    """Weights of the groups that receive rows, the gathered rows read, H written."""
    d, F, E, k = cfg["d_model"], cfg["d_ff"], cfg["n_experts"], cfg["top_k"]
    act = E if active_experts is None else active_experts
    T = cfg["batch"] * cfg["canvas_len"]
    rows = (k + 1) * T
    return (act + cfg["n_shared"]) * expert_group_bytes(cfg, "gateup") + rows * d * 2 + rows * F * 2


def gateup_flops_per_launch(cfg):
    """2 * rows * 2F * d over the shared expert's T rows and the k * T routed rows."""
    d, F, k = cfg["d_model"], cfg["d_ff"], cfg["top_k"]
    T = cfg["batch"] * cfg["canvas_len"]
    return 2 * (k + cfg["n_shared"]) * T * 2 * F * d


def gateup_roofline(cfg, avg_launch_ms, active_experts, peaks):
    """The gate/up GEMM against its own roofline: bytes over the measured copy
    bandwidth, or FLOPs over the measured sustained bf16 throughput, whichever
    takes longer for its algorithmic work."""
    nbytes = gateup_bytes_per_launch(cfg, active_experts)
    flops = gateup_flops_per_launch(cfg)
    t = avg_launch_ms / 1e3
    hbm, tflops, kind = peaks
    if flops / (tflops * 1e12) > nbytes / (hbm * 1e9):
        achieved = flops / t / 1e12
        return {"bound": "tensor", "kernel": "gemm_gateup", "achieved": achieved,
                "peak": tflops, "unit": "TFLOP/s", "frac": achieved / tflops,
                "peak_source": kind + " (sustained bf16)", "traffic": None,
                "algorithmic_flops_per_launch": flops, "avg_launch_ms": avg_launch_ms}
    achieved = nbytes / t / 1e9
    return {"bound": "hbm", "kernel": "gemm_gateup", "achieved": achieved, "peak": hbm,
            "unit": "GB/s", "frac": achieved / hbm, "peak_source": kind,
            "traffic": None if cfg.get("expert_fp8") else load_traffic("gemm_gateup", nbytes),
            "algorithmic_bytes_per_launch": nbytes, "avg_launch_ms": avg_launch_ms}


def flops_per_step(cfg):
    d, F, E, k = cfg["d_model"], cfg["d_ff"], cfg["n_experts"], cfg["top_k"]
    dh, Hq, Hkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    T = cfg["batch"] * cfg["canvas_len"]
    P, W, L, Tc = cfg["prompt_len"], cfg["window"], cfg["n_layers"], cfg["canvas_len"]
    f = 0
    for l in range(L):
        vis = P if (l + 1) % cfg["global_every"] == 0 else min(W, P)
        f += 2 * T * d * ((Hq + 2 * Hkv) * dh + Hq * dh + E)
        f += 4 * cfg["batch"] * Hq * Tc * (vis + Tc) * dh
        f += 2 * T * (k + 1) * 3 * F * d
    return f + 2 * T * d * cfg["vocab"]


# ----------------------------------------------------------------------------- peaks, clocks, traffic

def load_peaks():
    """(HBM GB/s, sustained bf16 TFLOP/s, "measured" | "fallback")."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return (float(j["hbm_gbs"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "measured")
    return 6650.0, 1400.0, "fallback"


def kernel_src_sha():
    """Hash of what the GEMM kernel is built from: gemm_tc.cu, gemm_shared.cuh,
    dg_common.cuh and the GemmArgs declaration (other declarations in dg_kernels.h
    do not count)."""
    csrc = os.path.join(ROOT, "canvas_denoising_step_b200", "csrc")
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "gemm_shared.cuh", "dg_common.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    hdr = open(os.path.join(csrc, "dg_kernels.h"), "rb").read()
    i = hdr.index(b"struct GemmArgs")
    h.update(hdr[i:hdr.index(b"};", i)])
    return h.hexdigest()[:16]


def load_traffic(kernel, algorithmic_bytes):
    """DRAM bytes per launch: the DRAM / algorithmic byte ratio of a committed ncu
    capture on a small case (one launch), times this launch's algorithmic bytes;
    None when the capture was not taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p)).get(kernel)
    if not j or j.get("kernel_src_sha") != kernel_src_sha():
        return None
    return j["dram_over_algorithmic"] * algorithmic_bytes


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms from before the
    timed region to after it; only the samples stamped inside the region are kept
    (the nearest later one when the region is shorter than the period)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        self.gpu = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.5)    # nvidia-smi is sampling before the region opens

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(text):
        import datetime
        try:
            return datetime.datetime.strptime(text.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.15)   # one more sample after the region closes
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 9]
        if not rows:
            return None
        stamped = [(self._stamp(r[0]), r) for r in rows]
        inside = [r for t, r in stamped if t is not None and self.t0 is not None and
                  self.t0 <= t <= self.t1]
        if not inside:
            later = [r for t, r in stamped if t is not None and self.t0 is not None and t >= self.t0]
            inside = later[:1] or rows[-1:]
        sm = [float(r[2]) for r in inside]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[6:10]) if "Active" in v and
                          "Not" not in v})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(inside[0][3]),
                "reasons": reasons, "samples": len(inside),
                "power_w_median": statistics.median(float(r[4]) for r in inside)}


# ----------------------------------------------------------------------------- CPU oracle timing

class _CachedWeights:
    """Oracle layer weights drawn once up front, so the timing excludes generation."""

    def __init__(self, oc, layer):
        from oracle import model as om
        self.W = om.layer_weights(oc, layer)
        for k in ("wq", "wk", "wv", "wo", "wr", "sg", "su", "sd"):
            self.W.get(k)
        self._experts = {e: self.W.expert(e) for e in range(oc.n_experts)}
        self.W.expert = self._experts.__getitem__


def oracle_sample(cfg, layers, vocab_fraction_den, seed_rows=0):
    """Time the oracle on a bounded sample of one pass: full-size layers `layers`
    (all 256 canvas rows) and a 1/vocab_fraction_den slice of the vocab head.
    Returns (seconds per layer list, seconds for the head slice)."""
    import numpy as np
    import synth
    from oracle import model as om
    oc = om.OracleConfig.from_dict(cfg)
    B, Tc, d = cfg["batch"], cfg["canvas_len"], cfg["d_model"]
    # with several canvases, one of them is run and the time scaled by the batch
    h = synth.hidden_states(cfg).float().numpy().astype(np.float64).reshape(B, Tc, d)[:1]
    bias = None
    if cfg.get("zipf_s"):
        bias = synth.zipf_router_bias(cfg["n_experts"], cfg["zipf_s"]).numpy()
    times = []
    for l in layers:
        Wc = _CachedWeights(oc, l)
        k, v = synth.prompt_kv(cfg, l)
        kp = k[:1].float().numpy().astype(np.float64)
        vp = v[:1].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        om.layer_forward(oc, Wc.W, h, kp, vp, router_bias=bias)
        times.append((time.perf_counter() - t0) * B)
    nv = cfg["vocab"] // vocab_fraction_den
    Eb = om.embedding_block(oc, 0, nv)
    hn = om.rmsnorm(h.reshape(Tc, d), 1.0, oc.rms_eps)
    t0 = time.perf_counter()
    lg = hn @ Eb.T
    om.logit_stats(lg, oc.mask_id)
    t_head = (time.perf_counter() - t0) * B
    return times, t_head


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg):
    """Oracle, as it stands, on a bounded sample of the workload: one local and one
    global layer at full size plus 1/32 of the vocab head; the pass time is
    extrapolated as 25 local + 5 global layers + 32 head slices."""
    L, ge = cfg["n_layers"], cfg["global_every"]
    n_glob = L // ge
    (t_loc, t_glob), t_head = oracle_sample(cfg, [0, ge - 1], 32)
    t_step = (L - n_glob) * t_loc + n_glob * t_glob + 32 * t_head
    value = cfg["batch"] * cfg["canvas_len"] / (cfg["steps"] * t_step)
    return {"value": value, "unit": "canvas tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"one local and one global full-size layer (256 canvas rows; times "
                       f"{cfg['batch']} for the batch) and 1/32 of the vocab head, weights "
                       f"pre-drawn; pass time extrapolated as "
                       f"{L - n_glob} local + {n_glob} global layers + 32 head slices "
                       f"= {t_step:.1f} s")}


# ----------------------------------------------------------------------------- arms

def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    L, ge = cfg["n_layers"], cfg["global_every"]
    per = []
    for s in range(args.warmup + args.steps):
        layer = ge - 1 if s % ge == ge - 1 else 0
        (t_l,), t_h = oracle_sample(cfg, [layer], L)
        if s >= args.warmup:
            per.append(L * (t_l + t_h))
    t_step = statistics.mean(per)
    value = cfg["batch"] * cfg["canvas_len"] / (cfg["steps"] * t_step)
    unit = "canvas tokens/s"
    line = {"metric": METRIC, "value": value,
            "unit": unit, "impl": "reference", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": (f"each step: one full-size oracle layer (local on 5 of 6 "
                                        f"steps, global on 1) plus 1/{L} of the vocab head, "
                                        f"weights pre-drawn, times {L}")},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def step_roofline(cfg, step_ms, active_avg, peaks):
    """A whole pass against max(bytes / HBM bandwidth, FLOPs / sustained bf16)."""
    hbm, tflops, _ = peaks
    nbytes = bytes_per_step(cfg, active_avg)
    flops = flops_per_step(cfg)
    t_hbm = nbytes / (hbm * 1e9) * 1e3
    t_tc = flops / (tflops * 1e12) * 1e3
    return {"bytes": nbytes, "flops": flops, "active_experts_per_layer": active_avg,
            "bytes_if_all_experts": bytes_per_step(cfg),
            "achieved_gbs": nbytes / (step_ms / 1e3) / 1e9,
            "frac_of_hbm": nbytes / (step_ms / 1e3) / 1e9 / hbm,
            "bound": "hbm" if t_hbm >= t_tc else "tensor",
            "roofline_ms": max(t_hbm, t_tc), "frac_of_roofline": max(t_hbm, t_tc) / step_ms}


def max_over_ranks(values, world, device):
    """Each timing taken as the maximum over the ranks (the slowest replica)."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def canvas_throughput(world, batch, canvas_len, steps, steps_per_block, t_ms):
    """Whole-job canvas tokens/s: every replica finalises batch * canvas_len tokens per
    steps_per_block passes; `steps` passes took t_ms (max over ranks)."""
    return world * batch * canvas_len * steps / steps_per_block / (t_ms / 1e3)


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import canvas_denoising_step_b200 as dg
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    B, Tc, S, L = cfg["batch"], cfg["canvas_len"], cfg["steps"], cfg["n_layers"]
    T = B * Tc
    with torch.cuda.stream(stream):
        ctx = dg.dg_create(dg.config_from_dict(cfg), stream.cuda_stream)
        dg.dg_init_weights(ctx, cfg["seed"])
        kv = []
        for l in range(L):
            k, v = synth.prompt_kv(cfg, l)
            kd, vd = k.to(dev, non_blocking=False), v.to(dev, non_blocking=False)
            kv.append((kd, vd))
            dg.dg_set_prompt_kv(ctx, l, kd.data_ptr(), vd.data_ptr(), B, cfg["prompt_len"])
        canvas0 = synth.initial_canvas(cfg).to(dev)
        canvas = canvas0.clone()
        if cfg.get("zipf_s"):
            bias = synth.zipf_router_bias(cfg["n_experts"], cfg["zipf_s"]).to(dev)
            dg.dg_set_router_bias(ctx, bias.data_ptr())
    stream.synchronize()

    def run_steps(n, start=0):
        for s in range(start, start + n):
            if s % S == 0:
                canvas.copy_(canvas0, non_blocking=True)
            dg.dg_canvas_step(ctx, canvas.data_ptr(), B, S - (s % S))

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
        dg.dg_sync(ctx)
        launches_per_step = dg.dg_last_launch_count(ctx)
        clocks = ClockSampler(local_rank)
        clocks.start()
        barrier()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.mark_begin()
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
        stream.synchronize()
        clocks.mark_end()
        clk = clocks.stop()
        barrier()
        ms = e0.elapsed_time(e1)
        dg.dg_sync(ctx)

        # per-kernel breakdown: a second pass of K steps with event records per launch
        dg.dg_profile_enable(ctx, 1)
        run_steps(args.steps)
        kern = {}
        i = 0
        while (name := dg.dg_kernel_name(i)) is not None:
            tot, cnt = dg.dg_profile_read(ctx, name)
            if cnt:
                kern[name] = (tot, cnt)
            i += 1
        dg.dg_profile_enable(ctx, 0)
        act = torch.empty(L, dtype=torch.int32, device=dev)
        dg.dg_debug_tensor(ctx, "expert_active", act.data_ptr(), 4 * L)
        active_avg = float(act.sum().item()) / (args.steps * L)

        # end to end through the host-buffer entry point
        hc = synth.initial_canvas(cfg).pin_memory()
        hconf = torch.empty(B, Tc).pin_memory()
        hcom = torch.empty(B, Tc, dtype=torch.uint8).pin_memory()
        h0 = hc.clone()
        for s in range(min(args.warmup, S)):
            dg.dg_canvas_step_host(ctx, hc.data_ptr(), B, S - s, hconf.data_ptr(), hcom.data_ptr())
        barrier()
        stream.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s in range(args.steps):
            if s % S == 0:
                hc.copy_(h0)
            dg.dg_canvas_step_host(ctx, hc.data_ptr(), B, S - (s % S), hconf.data_ptr(),
                                   hcom.data_ptr())
        f1.record(stream)
        stream.synchronize()
        ms_e2e = f0.elapsed_time(f1)
        barrier()

    t_max, t_e2e_max = max_over_ranks([ms, ms_e2e], world, dev)
    dg.dg_destroy(ctx)
    if rank != 0:
        return

    value = canvas_throughput(world, B, Tc, args.steps, S, t_max)
    peaks = load_peaks()
    peak = peaks[0]
    gu_ms, gu_n = kern.get("gemm_gateup", (float("nan"), 1))
    step_bytes = bytes_per_step(cfg, active_avg)
    step_ms = t_max / args.steps
    total_prof = sum(v[0] for v in kern.values())
    line = {
        "metric": METRIC,
        "value": value, "unit": "canvas tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_json(cfg, world),
        "roofline": gateup_roofline(cfg, gu_ms / gu_n, active_avg, peaks),
        "step_roofline": step_roofline(cfg, step_ms, active_avg, peaks),
        "kernels_ms_per_step": {k: v[0] / args.steps for k, v in
                                sorted(kern.items(), key=lambda kv: -kv[1][0])},
        "profiled_ms_per_step": total_prof / args.steps,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": canvas_throughput(world, B, Tc, args.steps, S, t_e2e_max),
                "unit": "canvas tokens/s",
                "h2d_bytes_per_step": T * 4, "d2h_bytes_per_step": T * 4 + T * 4 + T},
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    print(json.dumps(line), flush=True)


def layer_bytes(cfg, layer, active_experts):
    """Algorithmic HBM bytes of one block: its dense weights, the shared expert and the
    routed experts that receive rows, and the visible prompt K/V."""
    d, F, E = cfg["d_model"], cfg["d_ff"], cfg["n_experts"]
    dh, Hq, Hkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    P = cfg["prompt_len"]
    vis = P if (layer + 1) % cfg["global_every"] == 0 else min(cfg["window"], P)
    dense = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d)
    return dense + (active_experts + cfg["n_shared"]) * expert_group_bytes(cfg) + \
        2 * cfg["batch"] * Hkv * vis * dh * 2


def layer_flops(cfg, layer):
    d, F, E, k = cfg["d_model"], cfg["d_ff"], cfg["n_experts"], cfg["top_k"]
    dh, Hq, Hkv, Tc = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["canvas_len"]
    T = cfg["batch"] * Tc
    P = cfg["prompt_len"]
    vis = P if (layer + 1) % cfg["global_every"] == 0 else min(cfg["window"], P)
    return (2 * T * d * ((Hq + 2 * Hkv) * dh + Hq * dh + E) +
            4 * cfg["batch"] * Hq * Tc * (vis + Tc) * dh + 2 * T * (k + cfg["n_shared"]) * 3 * F * d)


def run_layer_case(args, cfg):
    """One decoder block (dg_layer_forward) on N(0,1) hidden states -- the
    single-layer workload -- timed with CUDA events over K calls after W warm-ups,
    with the clocks of the timed region, the per-kernel table, the block's roofline
    and the gate/up GEMM's, and the oracle timed on the same block."""
    import torch
    import canvas_denoising_step_b200 as dg
    import synth

    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    B, Tc, layer = cfg["batch"], cfg["canvas_len"], args.layer
    T = B * Tc
    with torch.cuda.stream(stream):
        ctx = dg.dg_create(dg.config_from_dict(cfg), stream.cuda_stream)
        dg.dg_init_weights(ctx, cfg["seed"])
        k, v = synth.prompt_kv(cfg, layer)
        kd, vd = k.cuda(), v.cuda()
        dg.dg_set_prompt_kv(ctx, layer, kd.data_ptr(), vd.data_ptr(), B, cfg["prompt_len"])
        x = synth.hidden_states(cfg).cuda()
        out = torch.empty_like(x)
        for _ in range(args.warmup):
            dg.dg_layer_forward(ctx, layer, x.data_ptr(), out.data_ptr(), T)
        dg.dg_sync(ctx)
        launches = dg.dg_last_launch_count(ctx)
        clocks = ClockSampler(0)
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        clocks.mark_begin()
        e0.record(stream)
        for _ in range(args.steps):
            dg.dg_layer_forward(ctx, layer, x.data_ptr(), out.data_ptr(), T)
        e1.record(stream)
        stream.synchronize()
        clocks.mark_end()
        clk = clocks.stop()
        ms = e0.elapsed_time(e1) / args.steps
        dg.dg_sync(ctx)
        act0 = torch.empty(cfg["n_layers"], dtype=torch.int32, device="cuda")
        dg.dg_debug_tensor(ctx, "expert_active", act0.data_ptr(), 4 * cfg["n_layers"])
        act_before = int(act0[layer].item())
        dg.dg_profile_enable(ctx, 1)
        for _ in range(args.steps):
            dg.dg_layer_forward(ctx, layer, x.data_ptr(), out.data_ptr(), T)
        kern, i = {}, 0
        while (name := dg.dg_kernel_name(i)) is not None:
            tot, cnt = dg.dg_profile_read(ctx, name)
            if cnt:
                kern[name] = (tot, cnt)
            i += 1
        dg.dg_profile_enable(ctx, 0)
        act = torch.empty(cfg["n_layers"], dtype=torch.int32, device="cuda")
        dg.dg_debug_tensor(ctx, "expert_active", act.data_ptr(), 4 * cfg["n_layers"])
        active = int(act[layer].item()) / args.steps
        dg.dg_destroy(ctx)
    del act_before
    peaks = load_peaks()
    hbm, tflops, kind = peaks
    nbytes, flops = layer_bytes(cfg, layer, active), layer_flops(cfg, layer)
    t_roof = max(nbytes / (hbm * 1e9), flops / (tflops * 1e12)) * 1e3
    gu_ms, gu_n = kern.get("gemm_gateup", (float("nan"), 1))
    line = {
        "metric": "decoder-block latency on 1 B200 (single-layer workload); % of its roofline",
        "value": ms, "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (f"one {'global' if (layer + 1) % cfg['global_every'] == 0 else 'local'} "
                                f"decoder block: d_model {cfg['d_model']}, {cfg['n_q_heads']}q/"
                                f"{cfg['n_kv_heads']}kv x {cfg['head_dim']}, {cfg['n_experts']} "
                                f"experts top-{cfg['top_k']} + {cfg['n_shared']} shared (width "
                                f"{cfg['d_ff']}), canvas {Tc} x batch {B}, prompt K/V "
                                f"{cfg['prompt_len']}, hidden states N(0,1), no vocab head"),
                   "name": cfg["name"], "layer": layer,
                   "l2": "inputs larger than L2: 1.6 GB of block weights per call",
                   "parallelism": "single"},
        "roofline": gateup_roofline(cfg, gu_ms / gu_n, active, peaks),
        "step_roofline": {"bytes": nbytes, "flops": flops, "active_experts": active,
                          "roofline_ms": t_roof, "frac_of_roofline": t_roof / ms,
                          "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                          "bound": "hbm" if nbytes / hbm / 1e9 >= flops / tflops / 1e12
                          else "tensor"},
        "kernels_ms_per_step": {k2: v2[0] / args.steps for k2, v2 in
                                sorted(kern.items(), key=lambda kv: -kv[1][0])},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline:
        (t_layer,), _ = oracle_sample(cfg, [layer], cfg["vocab"])
        line["cpu_baseline"] = {"value": t_layer * 1e3, "unit": "ms", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": "the same block on the same hidden states, in full "
                                          "(weights pre-drawn; the head term is one vocab row)"}
    print(json.dumps(line), flush=True)


def run_eb_case(args, cfg):
    """Entropy-bounded passes (dg_eb_step) on the workload: K passes after W warm-ups,
    each pass the whole stack, the head at the pass's temperature with the entropy
    reduction, the stop test and the bounded commit with its draw.  Reports the pass
    latency against the pass's roofline (the same bytes and FLOPs as a fixed-step
    pass: the entropy terms add no HBM traffic)."""
    import numpy as np
    import torch
    import canvas_denoising_step_b200 as dg
    import synth

    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    B, Tc, L = cfg["batch"], cfg["canvas_len"], cfg["n_layers"]
    n_max = 48
    with torch.cuda.stream(stream):
        ctx = dg.dg_create(dg.config_from_dict(cfg), stream.cuda_stream)
        dg.dg_init_weights(ctx, cfg["seed"])
        kv = []
        for l in range(L):
            k, v = synth.prompt_kv(cfg, l)
            kd, vd = k.cuda(), v.cuda()
            kv.append((kd, vd))
            dg.dg_set_prompt_kv(ctx, l, kd.data_ptr(), vd.data_ptr(), B, cfg["prompt_len"])
        g = np.random.default_rng(7)
        u = torch.from_numpy(g.uniform(size=(n_max, B, Tc)).astype(np.float32)).cuda()
        canvas0 = synth.initial_canvas(cfg).cuda()
        canvas = canvas0.clone()

        def passes(n):
            for s in range(n):
                step = s % n_max
                if step == 0:
                    canvas.copy_(canvas0, non_blocking=True)
                dg.dg_eb_step(ctx, canvas.data_ptr(), B, step, n_max,
                              u[step].data_ptr())

        passes(args.warmup)
        dg.dg_sync(ctx)
        launches = dg.dg_last_launch_count(ctx)
        clocks = ClockSampler(0)
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        clocks.mark_begin()
        e0.record(stream)
        passes(args.steps)
        e1.record(stream)
        stream.synchronize()
        clocks.mark_end()
        clk = clocks.stop()
        ms = e0.elapsed_time(e1) / args.steps
        dg.dg_sync(ctx)
        dg.dg_profile_enable(ctx, 1)
        passes(args.steps)
        kern, i = {}, 0
        while (name := dg.dg_kernel_name(i)) is not None:
            tot, cnt = dg.dg_profile_read(ctx, name)
            if cnt:
                kern[name] = tot / args.steps
            i += 1
        dg.dg_profile_enable(ctx, 0)
        act = torch.empty(L, dtype=torch.int32, device="cuda")
        dg.dg_debug_tensor(ctx, "expert_active", act.data_ptr(), 4 * L)
        active = float(act.sum().item()) / (args.steps * L)
        dg.dg_destroy(ctx)
    peaks = load_peaks()
    print(json.dumps({
        "metric": "entropy-bounded pass latency on 1 B200; % of the pass roofline",
        "value": ms, "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict(config_json(cfg, 1), sampler="entropy-bounded, 48 passes at most"),
        "step_roofline": step_roofline(cfg, ms, active, peaks),
        "kernels_ms_per_step": dict(sorted(kern.items(), key=lambda kv: -kv[1])),
        "gpu_launches": launches * args.steps, "clocks": clk}), flush=True)


def encoder_bytes(cfg, active_avg, chunk=None):
    """Algorithmic HBM bytes of encoding the workload's prompt (dg_encode) in chunks of
    `chunk` tokens (canvas_len by default): per chunk, every layer's weights the chunk
    needs once (q/k/v/o,
    router, the shared expert and `active_avg` routed experts per layer on average),
    the layer's visible cached K/V once (local layers: the window - 1 positions before
    the chunk at most) plus the chunk's own K/V appended, and the chunk's embedding rows."""
    d, E, L, B = cfg["d_model"], cfg["n_experts"], cfg["n_layers"], cfg["batch"]
    dh, Hq, Hkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    P, W = cfg["prompt_len"], cfg["window"]
    Tc = chunk or cfg["canvas_len"]
    dense = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d)
    n_chunks, kv = 0, 0
    for o in range(0, P, Tc):
        m = min(Tc, P - o)
        n_chunks += 1
        for l in range(L):
            vis = o if (l + 1) % cfg["global_every"] == 0 else min(W - 1, o)
            kv += 2 * B * Hkv * (vis + m) * dh * 2
    experts = n_chunks * L * (active_avg + cfg["n_shared"]) * expert_group_bytes(cfg)
    return n_chunks * L * dense + experts + kv + B * P * d * 2, n_chunks


def encoder_flops(cfg):
    """Algorithmic FLOPs of encoding the workload's prompt: per token and layer the
    q/k/v, o and router projections, the shared and top-k experts (gate, up, down),
    and causal attention QK^T and PV over the positions the token sees (all before it
    and itself on a global layer, the last `window` on a local one)."""
    d, F, E, k, L, B = (cfg["d_model"], cfg["d_ff"], cfg["n_experts"], cfg["top_k"],
                        cfg["n_layers"], cfg["batch"])
    dh, Hq, Hkv, P, W = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"], \
        cfg["prompt_len"], cfg["window"]
    per_token = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d) + \
        2 * (k + cfg["n_shared"]) * 3 * F * d
    total = 0
    for l in range(L):
        glob = (l + 1) % cfg["global_every"] == 0
        # sum over positions p of the keys p sees
        keys = P * (P + 1) // 2 if glob else \
            sum(min(p + 1, W) for p in range(P)) if P <= 4 * W else \
            W * (W + 1) // 2 + (P - W) * W
        total += B * (P * per_token + 2 * 2 * Hq * dh * keys)
    return total


def run_encode_case(args, cfg):
    """The causal encoder (dg_encode) over the workload's prompt: K encodings of
    prompt_len seeded random tokens per sequence from an empty context, after W
    warm-ups.  Reports encoded prompt tokens per second and the encoding against its
    HBM roofline (encoder_bytes)."""
    import numpy as np
    import torch
    import canvas_denoising_step_b200 as dg

    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    B, P, L, Tc = cfg["batch"], cfg["prompt_len"], cfg["n_layers"], cfg["canvas_len"]
    # room for up to 2048 rows a pass (as the batched workload): dg_encode takes chunks
    # of max_batch * canvas_len / batch tokens, and every chunk reads all the weights
    mb = max(B, min(2048 // Tc, B * -(-P // Tc)))
    with torch.cuda.stream(stream):
        ctx = dg.dg_create(dg.config_from_dict(cfg, max_batch=mb, max_context=P),
                           stream.cuda_stream)
        dg.dg_init_weights(ctx, cfg["seed"])
        g = np.random.default_rng(9)
        toks = torch.from_numpy(g.integers(1, cfg["vocab"], size=(B, P)).astype(np.int32)).cuda()

        def run(n):
            for _ in range(n):
                dg.dg_reset_context(ctx)
                dg.dg_encode(ctx, toks.data_ptr(), B, P)

        run(args.warmup)
        act = torch.empty(L, dtype=torch.int32, device="cuda")
        dg.dg_debug_tensor(ctx, "expert_active", act.data_ptr(), 4 * L)
        act0 = float(act.sum().item())
        clocks = ClockSampler(0)
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        clocks.mark_begin()
        e0.record(stream)
        run(args.steps)
        e1.record(stream)
        stream.synchronize()
        clocks.mark_end()
        clk = clocks.stop()
        ms = e0.elapsed_time(e1) / args.steps
        dg.dg_debug_tensor(ctx, "expert_active", act.data_ptr(), 4 * L)
        chunk = mb * Tc // B
        n_chunks = -(-P // chunk)
        active = (float(act.sum().item()) - act0) / (args.steps * n_chunks * L)
        # per-kernel times: one more round with every launch bracketed by events
        dg.dg_profile_enable(ctx, 1)
        run(args.steps)
        kern, i = {}, 0
        while (name := dg.dg_kernel_name(i)) is not None:
            tot, cnt = dg.dg_profile_read(ctx, name)
            if cnt:
                kern[name] = tot / args.steps
            i += 1
        dg.dg_profile_enable(ctx, 0)
        dg.dg_destroy(ctx)
    peaks = load_peaks()
    nbytes, _ = encoder_bytes(cfg, active, chunk)
    flops = encoder_flops(cfg)
    hbm, tflops = peaks[0], peaks[1]
    bytes_ms = nbytes / (hbm * 1e9) * 1e3
    flops_ms = flops / (tflops * 1e12) * 1e3
    roof_ms = max(bytes_ms, flops_ms)
    print(json.dumps({
        "metric": "encoded prompt tokens/sec on 1 B200 (causal encoder); % of its HBM roofline",
        "value": B * P / (ms / 1e3), "unit": "prompt tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(config_json(cfg, 1),
                                            case=f"encode {P} random prompt tokens per sequence "
                                                 f"in chunks of {chunk}"),
        "encode_roofline": {"bytes": nbytes, "flops": flops,
                            "active_experts_per_layer_chunk": active,
                            "bytes_ms": bytes_ms, "flops_ms": flops_ms, "roofline_ms": roof_ms,
                            "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                            "achieved_tflops": flops / (ms / 1e3) / 1e12,
                            "frac_of_roofline": roof_ms / ms,
                            "bound": "tensor" if flops_ms > bytes_ms else "hbm",
                            "peak": tflops if flops_ms > bytes_ms else hbm,
                            "peak_source": peaks[2]},
        "kernels_ms_per_step": dict(sorted(kern.items(), key=lambda kv: -kv[1])),
        "clocks": clk}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["step", "layer", "encode"], default="step",
                    help="step: full canvas passes (the headline); layer: dg_layer_forward; "
                         "encode: the causal encoder over the prompt")
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--sampler", choices=["fixed", "eb"], default="fixed",
                    help="fixed: k = ceil(r / steps_left) commits (the headline); eb: "
                         "entropy-bounded passes")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=INT",
                    help="override an integer workload field (kernel studies only)")
    args = ap.parse_args()
    if args.warmup < 3 and args.case == "step":
        ap.error("--warmup must be >= 3")
    import synth
    cfg = synth.config(args.workload, **{kv.split("=")[0]: int(kv.split("=")[1])
                                         for kv in args.set})
    if args.case == "layer":
        run_layer_case(args, cfg)
        return
    if args.case == "encode":
        run_encode_case(args, cfg)
        return
    if args.sampler == "eb":
        run_eb_case(args, cfg)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, cfg, rank, world)
        else:
            run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1 and args.impl == "ours":
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
