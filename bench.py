#!/usr/bin/env python3
"""Benchmark of the MoE FFN block forward pass on B200: MoE-layer tokens/s and the fraction
of the HBM / bf16 roofline reached.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|keras|zipf|chain]
                    [--impl ours|reference] [--eager]

Workloads (seeded synthetic inputs of the block's standard configurations):
  decode   (default) D=2048, E=128, k=8, I=768; one step = one block pass for each of
           T = 1, 8, 32, 128, 256 tokens (425 tokens per step);
  prefill  same shape, T = 8192;
  keras    D=2048, E=60, k=4, I=1408, T=4096;
  zipf     D=2048, E=512, k=10, I=512 + gated shared expert (I_s=512), Zipf(1.1) router bias;
  chain    48 residual blocks of the keras shape, T=4096 (weights drawn on the GPU).
Inputs are resident in HBM when the timed region starts.  Decode weights rotate through one
copy per T so every pass streams its experts from HBM (each copy 1.2 GB > 126 MB L2); the
other workloads' weights and activations exceed L2 by themselves.

Timing: W untimed warm-up steps, then K steps captured as CUDA graphs (one untimed upload
replay), timed with CUDA events on the launch stream between a barrier and a device
synchronise on both sides; max over ranks.  That replay gives the headline value.  A second
timed replay of the same K steps, captured with six stage events per block pass (start,
routed, permuted, gate_up, down, combined), gives each stage's duration and the dominant
kernel's roofline (event nodes between kernels cost a little time, so they are kept out of
the headline replay).  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (1 B200) at D=2048,E=128,k=8,I=768; % of HBM/bf16 roofline"

WORKLOADS = {
    "decode": dict(config="decode", sweep=(1, 8, 32, 128, 256), layers=1),
    "prefill": dict(config="prefill", sweep=(8192,), layers=1),
    "keras": dict(config="keras", sweep=(4096,), layers=1),
    "zipf": dict(config="zipf", sweep=(4096,), layers=1),
    "chain": dict(config="keras", sweep=(4096,), layers=48),
}

FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)

NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
}


# ------------------------------------------------------------------ helpers (no GPU needed)

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d["bf16_tflops_sustained"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def aggregate(per_rank_ms, tokens_per_step_per_rank, steps, world):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    t = max(per_rank_ms)
    return dict(ms=t, ms_per_step=t / steps, value=world * tokens_per_step_per_rank * steps / (t / 1e3))


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def profile_traffic(kernel_tag):
    """Per-launch DRAM traffic of a kernel from the committed ncu summary, if the summary was
    taken on the kernel source as it is now (its recorded sha256 matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})\s+(\S+)", text)
    if not m or not h:
        return None
    try:
        src = open(os.path.join(ROOT, h.group(2)), "rb").read()
    except OSError:
        return None
    if hashlib.sha256(src).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


def kernels_per_forward(T, k, streaming):
    """Kernels one moe_forward_ex call launches (the library's launch sequence): T <= 32 one
    fused routing + permutation kernel; above, the router, then selection + permutation in
    one kernel while T*k <= 4096 (else selection, histogram, scan and scatter), and the
    permuted copy of x for the grouped path; then gate_up, down and the combine."""
    n = 0
    if T <= 32:
        n += 1
    else:
        n += 1 + (1 if T * k <= 4096 else 4)
        n += 0 if streaming else 1
    return n + 3


class ClockSampler:
    """Samples the SM clock and clock-event reasons of one GPU through NVML while running."""

    def __init__(self, torch_device_index=0, period_s=0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid if not uuid.startswith("GPU-") else uuid)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[torch_device_index]) if vis and vis.split(",")[0].isdigit() else torch_device_index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvml unavailable"], samples=0)
        names = [n for b, n in NVML_REASONS.items() if self.reasons & b]
        return dict(sm_mhz=statistics.median(self.samples) if self.samples else None,
                    sm_max_mhz=self.max_mhz, reasons=names, samples=len(self.samples))


# ------------------------------------------------------------------ workload

def build_workload(args, device):
    import torch
    from sparse_fp32_softmax_b200 import inputs
    spec = WORKLOADS[args.workload]
    cfg = inputs.CONFIGS[spec["config"]]
    sweep = spec["sweep"]
    Tmax = max(sweep)
    W = []
    if spec["layers"] > 1:
        for l in range(spec["layers"]):
            W.append(inputs.make_layer(cfg, T=Tmax, layer=l, device=device, gen_device=device, with_x=False))
        x0 = inputs.normal_bf16((Tmax, cfg.D), 1.0, 1000 * cfg.seed + inputs.TID_X).to(device)
    else:
        L = inputs.make_layer(cfg, T=Tmax)
        x0 = L["x"].to(device)
        base = {k: (v.to(device) if v is not None else None) for k, v in L.items() if k != "x"}
        W.append(base)
        copies = len(sweep) if args.copies is None else max(1, args.copies)
        for _ in range(1, copies):              # one weight copy per pass of a step
            W.append({k: (v.clone() if v is not None else None) for k, v in base.items()})
    return cfg, spec, sweep, W, x0


def passes_of(cfg, spec, sweep, W, x0, torch):
    """The block passes of one step: (T, x, weights, residual-source index)."""
    ps = []
    if spec["layers"] > 1:
        for l in range(spec["layers"]):
            ps.append(dict(T=sweep[0], layer=l, w=W[l]))
    else:
        for i, T in enumerate(sweep):
            ps.append(dict(T=T, layer=None, w=W[i % len(W)], x=x0[:T].contiguous()))
    return ps


def run_ours(args, rank, world, device):
    import torch
    from sparse_fp32_softmax_b200 import binding as B
    from sparse_fp32_softmax_b200.roofline import algorithmic_bytes, algorithmic_flops

    cfg, spec, sweep, W, x0 = build_workload(args, device)
    chain = spec["layers"] > 1
    passes = passes_of(cfg, spec, sweep, W, x0, torch)
    path = args.path
    stream = torch.cuda.current_stream()

    # per-pass buffers, workspaces and routing outputs
    act = [torch.empty_like(x0), torch.empty_like(x0)] if chain else None
    shared_ws = None
    for n, p in enumerate(passes):
        T = p["T"]
        w = p["w"]
        p["dims"] = B.make_dims(T, cfg.D, cfg.E, cfg.k, cfg.I, cfg.norm_topk_prob)
        p["idx"] = torch.empty(T, cfg.k, dtype=torch.int32, device=device)
        if chain:                               # x0 -> A -> B -> A ...; x0 is never written
            p["x"] = x0 if n == 0 else act[(n - 1) % 2]
            p["out"] = act[n % 2]
            p["residual"] = p["x"]
        else:
            p["out"] = torch.empty_like(p["x"])
            p["residual"] = None
        opts = B.make_opts(router_bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                           shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"),
                           residual=p["residual"], topk_idx_out=p["idx"], path=path)
        p["opts_base"] = opts
        if chain:                               # passes run one after another: one workspace
            if shared_ws is None:
                shared_ws = B.workspace(p["dims"], opts, device=device)
            p["ws"] = shared_ws
        else:
            p["ws"] = B.workspace(p["dims"], opts, device=device)

    def enqueue(p, events=None):
        w = p["w"]
        opts = B.make_opts(router_bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                           shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"),
                           residual=p["residual"], topk_idx_out=p["idx"], path=path,
                           stage_events=events)
        B.moe_forward_ex(p["x"], w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, cfg.norm_topk_prob,
                         out=p["out"], ws=p["ws"], opts=opts)

    def step(events_for_step=None):
        for n, p in enumerate(passes):
            enqueue(p, events_for_step[n] if events_for_step else None)

    # warm-up (also settles routing for the byte accounting)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for p in passes:
        assert B.moe_get_device_status(p["ws"]) == B.MOE_OK
        counts = torch.bincount(p["idx"].reshape(-1).long(), minlength=cfg.E)
        p["touched"] = int((counts > 0).sum())
        p["max_load"] = int(counts.max())
        p["streaming"] = (path == "stream")

    K = args.steps
    evs = [[B.stage_events(6) for _ in passes] for _ in range(K)]
    use_graph = not args.eager

    def capture(with_events):
        graphs = []
        chunk = 25
        for c0 in range(0, K, chunk):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=torch.cuda.Stream(device=device)):
                for s in range(c0, min(K, c0 + chunk)):
                    step(evs[s] if with_events else None)
            graphs.append(g)
        for g in graphs:                       # untimed upload replay
            g.replay()
        torch.cuda.synchronize()
        return graphs

    if world > 1:
        import torch.distributed as dist

    def timed(graphs, with_events, sampler=None):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if sampler:
            sampler.__enter__()
        start.record()
        if graphs is not None:
            for g in graphs:
                g.replay()
        else:
            for s in range(K):
                step(evs[s] if with_events else None)
        end.record()
        torch.cuda.synchronize()
        if sampler:
            sampler.__exit__(None, None, None)
        if world > 1:
            dist.barrier()
        return start.elapsed_time(end)

    sampler = ClockSampler(torch.cuda.current_device())
    ms = timed(capture(False) if use_graph else None, False, sampler)
    ms_events = timed(capture(True) if use_graph else None, True)
    per_rank = [ms]
    if world > 1:
        t = torch.tensor([ms], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        per_rank = [float(t.item())]
    tokens_per_step = sum(p["T"] for p in passes) if not chain else sweep[0]
    agg = aggregate(per_rank, tokens_per_step, K, world)

    # stage durations of every pass of every timed step
    stage_ms = [[0.0] * 5 for _ in passes]
    for s in range(K):
        for n in range(len(passes)):
            e = evs[s][n]
            for j in range(5):
                stage_ms[n][j] += e[j].elapsed_time(e[j + 1]) / K
    peaks = load_peaks()
    launches_per_pass = [kernels_per_forward(p["T"], cfg.k, p["streaming"]) for p in passes]

    # roofline of the dominant kernel: the gate_up expert kernel (stage 3).  Reported for
    # the workload's largest pass (one launch shape, the one a single ncu capture covers);
    # every pass's gate_up rate is listed in the sweep entries.
    I2 = 2 * cfg.I
    blk_bytes = blk_flops = 0.0
    per_T = []
    gu = []
    for n, p in enumerate(passes):
        T = p["T"]
        b_gu = p["touched"] * I2 * cfg.D * 2 + (2 * cfg.I_s * cfg.D * 2 if cfg.I_s else 0)
        f_gu = 2.0 * T * cfg.k * I2 * cfg.D + (2.0 * T * 2 * cfg.I_s * cfg.D if cfg.I_s else 0)
        gu.append((b_gu, f_gu, stage_ms[n][2]))
        b = algorithmic_bytes(T, cfg.D, cfg.E, cfg.k, cfg.I, p["touched"], cfg.I_s, cfg.shared_gated,
                              residual=chain)
        f = algorithmic_flops(T, cfg.D, cfg.E, cfg.k, cfg.I, cfg.I_s, cfg.shared_gated)
        blk_bytes += b
        blk_flops += f
        t_pass = sum(stage_ms[n])
        t_roof = max(b / (peaks["hbm_gbs"] * 1e9), f / (peaks["bf16_tflops_sustained"] * 1e12))
        if not chain:
            per_T.append(dict(T=T, us=round(t_pass * 1e3, 2), tokens_per_s=round(T / (t_pass / 1e3), 1),
                              roofline_us=round(t_roof * 1e6, 2), roofline_frac=round(t_roof / (t_pass / 1e3), 4),
                              touched=p["touched"], max_load=p["max_load"],
                              stages_us=[round(v * 1e3, 2) for v in stage_ms[n]],
                              gate_up_gbs=round(b_gu / (stage_ms[n][2] / 1e3) / 1e9, 1),
                              gate_up_tflops=round(f_gu / (stage_ms[n][2] / 1e3) / 1e12, 1),
                              path="stream" if p["streaming"] else "grouped"))
    gu_bytes, gu_flops, gu_ms = gu[-1]
    if chain:   # every layer has the same shape: average them
        gu_bytes = sum(g[0] for g in gu) / len(gu)
        gu_flops = sum(g[1] for g in gu) / len(gu)
        gu_ms = sum(g[2] for g in gu) / len(gu)
    # the bound follows the kernel's own work: weight bytes at HBM peak against FLOPs at the
    # sustained bf16 peak (decode is weight-bound, prefill compute-bound)
    t_bytes = gu_bytes / (peaks["hbm_gbs"] * 1e9)
    t_flops = gu_flops / (peaks["bf16_tflops_sustained"] * 1e12)
    streaming = all(p["streaming"] for p in passes)
    kname = "stream_gate_up_kernel" if streaming else "tc_gemm_kernel<gate_up>"
    T_dom = passes[-1]["T"]
    if t_bytes >= t_flops:
        achieved = gu_bytes / (gu_ms / 1e3) / 1e9
        roof = dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=round(achieved / peaks["hbm_gbs"], 4), kernel=kname, launch=f"T={T_dom}",
                    algorithmic_bytes_per_launch=int(gu_bytes),
                    peak_source=peaks["source"] + " hbm_gbs")
    else:
        achieved = gu_flops / (gu_ms / 1e3) / 1e12
        roof = dict(bound="tensor", achieved=round(achieved, 1), peak=peaks["bf16_tflops_sustained"],
                    unit="TFLOP/s", frac=round(achieved / peaks["bf16_tflops_sustained"], 4),
                    kernel=kname, launch=f"T={T_dom}", algorithmic_flops_per_launch=int(gu_flops),
                    peak_source=peaks["source"] + " bf16_tflops_sustained")
    tag = ("stream_gate_up_" if streaming else "tc_gate_up_") + args.workload
    if tag == "tc_gate_up_prefill":
        tag = "tc_gemm_prefill"
    # DRAM bytes of one launch from the committed ncu summary (null when there is none for
    # this workload or the kernel source changed since it was taken)
    roof["traffic"] = profile_traffic(tag)
    blk_time = max(blk_bytes / (peaks["hbm_gbs"] * 1e9), blk_flops / (peaks["bf16_tflops_sustained"] * 1e12))

    # end to end through the public API with host buffers (eager, copies inside the region)
    e2e = None
    if not chain:
        hx = [p["x"].cpu().pin_memory() for p in passes]
        hy = [torch.empty(p["out"].shape, dtype=p["out"].dtype).pin_memory() for p in passes]
        dx = [torch.empty_like(p["x"]) for p in passes]

        def e2e_step():
            for n, p in enumerate(passes):
                dx[n].copy_(hx[n], non_blocking=True)
                w = p["w"]
                B.moe_forward_ex(dx[n], w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, cfg.norm_topk_prob,
                                 out=p["out"], ws=p["ws"], opts=p["opts_base"])
                hy[n].copy_(p["out"], non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(K):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e_ms = s0.elapsed_time(s1)
        if world > 1:
            t = torch.tensor([e_ms], device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        bytes_in = sum(p["x"].numel() * 2 for p in passes)
        e2e = dict(value=round(world * tokens_per_step * K / (e_ms / 1e3), 1), unit="tokens/s",
                   h2d_bytes_per_step=bytes_in, d2h_bytes_per_step=bytes_in, timing="eager")

    line = dict(
        metric=METRIC, value=round(agg["value"], 1), unit="tokens/s", n_gpus=world, steps=K,
        warmup=args.warmup, ms_per_step=round(agg["ms_per_step"], 5), higher_is_better=True,
        scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
        config=dict(workload=describe(args.workload, cfg, sweep, spec), tokens_per_step=tokens_per_step,
                    stage_timing=f"second timed replay of the {K} steps with stage events: "
                                 f"{ms_events / K:.4f} ms/step",
                    l2=("rotating %d weight copies (%.1f GB) > 126 MB L2" % (len(W), len(W) * weight_gb(cfg))
                        if not chain else "48 distinct layers (%.1f GB) > 126 MB L2" % (48 * weight_gb(cfg))),
                    timing="CUDA graph replay" if use_graph else "eager", path=path,
                    parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        roofline=roof,
        block_roofline=dict(time_us=round(blk_time * 1e6, 2), measured_us=round(agg["ms_per_step"] * 1e3, 2),
                            frac=round(blk_time / (agg["ms_per_step"] / 1e3), 4),
                            bytes=int(blk_bytes), flops=int(blk_flops)),
        gpu_launches=int(sum(launches_per_pass) * K),
        clocks=sampler.summary(),
        e2e=e2e,
    )
    if per_T:
        line["sweep"] = per_T
    return line, cfg, passes


def weight_gb(cfg):
    return (cfg.E * 3 * cfg.D * cfg.I * 2 + cfg.E * cfg.D * 2 + 3 * cfg.D * cfg.I_s * 2) / 1e9


def describe(name, cfg, sweep, spec):
    s = (f"{name}: D={cfg.D}, E={cfg.E}, k={cfg.k}, I={cfg.I}, norm_topk_prob={cfg.norm_topk_prob}, "
         f"T={'/'.join(str(t) for t in sweep)}")
    if cfg.I_s:
        s += f", gated shared expert I_s={cfg.I_s}"
    if cfg.zipf_s:
        s += f", Zipf({cfg.zipf_s}) router bias"
    if spec["layers"] > 1:
        s += f", {spec['layers']} residual blocks"
    return s + "; x ~ N(0,1), weights ~ N(0,0.02), bf16, seeded"


# ------------------------------------------------------------------ CPU oracle legs

def oracle_sample_rate(cfg, x, w, rows, threads):
    """Oracle tokens/s over `rows` with `threads` threads (one forward per row)."""
    from oracle import oracle as O
    t0 = time.perf_counter()
    O.forward_rows(x, w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, rows, norm=cfg.norm_topk_prob,
                   bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                   shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"), threads=threads)
    return len(rows) / (time.perf_counter() - t0)


def cpu_baseline(cfg, target_cpu_s=10.0, layers=1):
    """The oracle as it stands on this host's cores, on a bounded sample of the workload."""
    from oracle import oracle as O
    from sparse_fp32_softmax_b200 import inputs
    L = inputs.make_layer(cfg, T=cfg.T)
    threads = O.cpu_threads_available()
    one = oracle_sample_rate(cfg, L["x"], L, [0], 1)           # seconds per token on one core
    n = int(max(threads, min(2048, target_cpu_s * one)))
    n = min(n, cfg.T)
    rows = list(range(n))
    rate = oracle_sample_rate(cfg, L["x"], L, rows, threads) / layers
    return dict(value=round(rate, 3), unit="tokens/s", cores=threads, kind="oracle",
                sample=f"first {n} tokens of the T={cfg.T} batch, one FP64 block pass each "
                       f"(~{n / one:.0f} CPU-seconds)" + (f", rate divided by {layers} layers" if layers > 1 else ""))


def run_reference(args):
    """The oracle timed as the reference arm: each step is a bounded sample of the workload."""
    from oracle import oracle as O
    from sparse_fp32_softmax_b200 import inputs
    spec = WORKLOADS[args.workload]
    cfg = inputs.CONFIGS[spec["config"]]
    sweep = spec["sweep"]
    L = inputs.make_layer(cfg, T=max(sweep))
    threads = O.cpu_threads_available()
    rows = list(range(min(threads, max(sweep))))             # one token per core per step
    for _ in range(args.warmup):
        oracle_sample_rate(cfg, L["x"], L, rows, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_rate(cfg, L["x"], L, rows, threads)
    dt = time.perf_counter() - t0
    value = len(rows) * args.steps / dt * spec["layers"] ** -1
    return dict(metric=METRIC, value=round(value, 3), unit="tokens/s", n_gpus=1, steps=args.steps,
                warmup=args.warmup, ms_per_step=round(dt / args.steps * 1e3, 3), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=describe(args.workload, cfg, sweep, spec),
                            sample=f"{len(rows)} tokens of the T={max(sweep)} batch per step"),
                cpu_baseline=dict(value=round(value, 3), unit="tokens/s", cores=threads, kind="oracle",
                                  sample=f"{len(rows)} tokens per step, {args.steps} steps"),
                e2e=dict(value=round(value, 3), unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "stream", "grouped"])
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=None,
                    help="decode weight copies in rotation (default: one per pass of a step)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"impl": "ours", "error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    from sparse_fp32_softmax_b200.build import build
    build()
    line, cfg, _ = run_ours(args, rank, world, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, layers=WORKLOADS[args.workload]["layers"])
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
