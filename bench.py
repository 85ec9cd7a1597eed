#!/usr/bin/env python3
"""Benchmark of the MoE FFN block forward pass on B200: MoE-layer tokens/s and the fraction
of the HBM / bf16 roofline reached.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|keras|zipf|chain]
                    [--extra prefill,keras,zipf,chain|none] [--impl ours|reference] [--eager]
                    [--sweep T[,T...]]

Workloads (seeded synthetic inputs of the block's standard configurations):
  decode   (headline) D=2048, E=128, k=8, I=768; one step = one block pass for each of
           T = 1, 8, 32, 128, 256 tokens (425 tokens per step);
  prefill  same shape, T = 8192;
  keras    D=2048, E=60, k=4, I=1408, T=4096;
  zipf     D=2048, E=512, k=10, I=512 + gated shared expert (I_s=512), Zipf(1.1) router bias;
  chain    48 residual blocks of the keras shape, T=4096 (weights drawn on the GPU).
The headline workload gives the JSON line's value; the ``--extra`` workloads (by default
prefill, keras, zipf and chain) are measured in the same run and reported under
"workloads", each with its own roofline, block fraction and CPU baseline.
Inputs are resident in HBM when a timed region starts.  Decode weights rotate through one
copy per pass so every pass streams its experts from HBM (each copy 1.2 GB > 126 MB L2); the
other workloads' weights and activations exceed L2 by themselves.

Timing: W untimed warm-up steps, then K steps captured as CUDA graphs (one untimed upload
replay), timed with CUDA events on the launch stream between a barrier and a device
synchronise on both sides; max over ranks.  That replay gives the value.  For a sweep,
each T is also timed alone the same way (K passes, rotating the weight copies).  A second
timed replay of the K steps, captured with six stage events per block pass (start, routed,
permuted, gate_up, down, combined), gives each stage's duration and the per-kernel
rooflines (event nodes between kernels cost a little time, so they are kept out of the
other timings).  Roofline peaks: the measured burst bf16 figure for timed regions under a
second, the sustained one for longer regions.  ``--impl reference`` times the CPU oracle
instead (rank 0 only).
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
    # the decode sweep with FP8 E4M3 weight-only experts (per-row scales, quantised by the
    # library); its roofline counts one byte per expert weight plus the scales
    "decode_fp8": dict(config="decode", sweep=(1, 8, 32, 128, 256), layers=1, fp8=True),
}
DEFAULT_EXTRA = "prefill,keras,zipf,chain,decode_fp8"

FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)
SUSTAINED_REGION_S = 1.0     # timed regions at least this long divide by the sustained peak

NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
}

# stage k of the stage events (between event k and k+1)
STAGES = ("route", "permute", "gate_up", "down", "combine")


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


def tensor_peak(peaks, region_s):
    """(TFLOP/s, name) of the bf16 peak a kernel timed inside a region of region_s seconds is
    held to: the burst figure for short regions, the sustained one for long ones."""
    if region_s >= SUSTAINED_REGION_S:
        return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return peaks["bf16_tflops"], "bf16_tflops"


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


def kernels_per_forward(T, k, path="grouped"):
    """Kernels one moe_forward_ex call launches (the library's launch sequence): on the decode
    path one; on the grouped path the router; selection + permutation in one kernel while
    T*k <= 4096, else selection, histogram, scan and scatter; for T > 32 the permuted copy of
    x; then gate_up, down and the combine."""
    if path == "decode":
        return 1
    return 1 + (1 if T * k <= 4096 else 4) + (1 if T > 32 else 0) + 3


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


# ------------------------------------------------------------------ workload

def build_workload(name, device, copies=None):
    """(cfg, spec, sweep, device weight sets, device x, CPU layer or None)."""
    import torch
    from sparse_fp32_softmax_b200 import inputs
    spec = WORKLOADS[name]
    cfg = inputs.CONFIGS[spec["config"]]
    sweep = spec["sweep"]
    Tmax = max(sweep)
    W = []
    L = None
    if spec["layers"] > 1:
        for l in range(spec["layers"]):
            W.append(inputs.make_layer(cfg, T=Tmax, layer=l, device=device, gen_device=device, with_x=False))
        x0 = inputs.normal_bf16((Tmax, cfg.D), 1.0, 1000 * cfg.seed + inputs.TID_X).to(device)
    else:
        L = inputs.make_layer(cfg, T=Tmax)
        x0 = L["x"].to(device)
        base = {k: (v.to(device) if v is not None else None) for k, v in L.items() if k != "x"}
        W.append(base)
        n = len(sweep) if copies is None else max(1, copies)
        for _ in range(1, n):              # one weight copy per pass of a step
            W.append({k: (v.clone() if v is not None else None) for k, v in base.items()})
    if spec.get("fp8"):
        from sparse_fp32_softmax_b200 import binding as B
        for w in W:                        # FP8 experts replace the bf16 ones
            q_gu, s_gu = B.moe_quantize_fp8_rows(w.pop("W_gate_up"))
            q_dn, s_dn = B.moe_quantize_fp8_rows(w.pop("W_down"))
            w["W_gate_up"] = w["W_down"] = None
            w["fp8"] = dict(W_gate_up_fp8=q_gu, gate_up_scale=s_gu, W_down_fp8=q_dn, down_scale=s_dn)
        torch.cuda.synchronize()
    return cfg, spec, sweep, W, x0, L


def measure(name, args, rank, world, device, peaks, with_e2e):
    """Time one workload; returns (result dict, cfg, CPU layer)."""
    import ctypes

    import torch
    from sparse_fp32_softmax_b200 import binding as B
    from sparse_fp32_softmax_b200 import inputs
    from sparse_fp32_softmax_b200.roofline import algorithmic_bytes, algorithmic_flops

    cfg, spec, sweep, W, x0, L_cpu = build_workload(name, device, args.copies if name == args.workload else None)
    chain = spec["layers"] > 1
    K = args.steps
    if world > 1:
        import torch.distributed as dist

    # the block passes of one step, with their buffers and workspaces
    passes = []
    if chain:
        act = [torch.empty_like(x0), torch.empty_like(x0)]
        for l in range(spec["layers"]):       # x0 -> A -> B -> A ...; x0 is never written
            passes.append(dict(T=sweep[0], w=W[l], x=x0 if l == 0 else act[(l - 1) % 2], out=act[l % 2]))
            passes[-1]["residual"] = passes[-1]["x"]
    else:
        for i, T in enumerate(sweep):
            passes.append(dict(T=T, w=W[i % len(W)], x=x0[:T].contiguous(), residual=None))
            passes[-1]["out"] = torch.empty_like(passes[-1]["x"])
    shared_ws = None
    for p in passes:
        w = p["w"]
        p["dims"] = B.make_dims(p["T"], cfg.D, cfg.E, cfg.k, cfg.I, cfg.norm_topk_prob)
        p["idx"] = torch.empty(p["T"], cfg.k, dtype=torch.int32, device=device)
        p["opts"] = B.make_opts(router_bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                                shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"),
                                residual=p["residual"], topk_idx_out=p["idx"], **w.get("fp8", {}))
        p["path"] = B.moe_forward_path(p["dims"], p["opts"])
        if chain:                             # passes run one after another: one workspace
            if shared_ws is None:
                shared_ws = B.workspace(p["dims"], p["opts"], device=device)
            p["ws"] = shared_ws
        else:
            p["ws"] = B.workspace(p["dims"], p["opts"], device=device)

    def enqueue(p, w=None, events=None):
        w = p["w"] if w is None else w
        opts = p["opts"]
        if events is not None:
            opts = B.make_opts(router_bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                               shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"),
                               residual=p["residual"], topk_idx_out=p["idx"], stage_events=events,
                               **w.get("fp8", {}))
        B.moe_forward_ex(p["x"], w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, cfg.norm_topk_prob,
                         out=p["out"], ws=p["ws"], opts=opts)

    def step(events_for_step=None):
        for n, p in enumerate(passes):
            enqueue(p, events=events_for_step[n] if events_for_step else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for p in passes:
        assert B.moe_get_device_status(p["ws"]) == B.MOE_OK
        counts = torch.bincount(p["idx"].reshape(-1).long(), minlength=cfg.E)
        p["touched"] = int((counts > 0).sum())
        p["max_load"] = int(counts.max())

    use_graph = not args.eager
    evs = [[B.stage_events(6) for _ in passes] for _ in range(K)]

    def capture(body, n):
        """CUDA graphs of body(s) for s in range(n), in chunks; one untimed upload replay."""
        graphs = []
        chunk = max(1, 1000 // max(1, len(passes)))
        for c0 in range(0, n, chunk):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=torch.cuda.Stream(device=device)):
                for s in range(c0, min(n, c0 + chunk)):
                    body(s)
            graphs.append(g)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        return graphs

    def timed(graphs, eager_body, n, sampler=None):
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
            for s in range(n):
                eager_body(s)
        end.record()
        torch.cuda.synchronize()
        if sampler:
            sampler.__exit__(None, None, None)
        if world > 1:
            dist.barrier()
        ms = start.elapsed_time(end)
        if world > 1:
            t = torch.tensor([ms], device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms

    def run(body, n, sampler=None):
        graphs = capture(body, n) if use_graph else None
        ms = timed(graphs, body, n, sampler)
        del graphs
        return ms

    sampler = ClockSampler(torch.cuda.current_device())
    ms = run(lambda s: step(), K, sampler)
    ms_events = run(lambda s: step(evs[s]), K)
    tokens_per_step = sweep[0] if chain else sum(p["T"] for p in passes)
    agg = aggregate([ms], tokens_per_step, K, world)
    # each T of a sweep alone (K passes, the weight copies in rotation)
    per_T_ms = {}
    if len(passes) > 1:
        for n, p in enumerate(passes):
            per_T_ms[p["T"]] = run(lambda s, p=p: enqueue(p, w=W[s % len(W)]), K) / K

    # stage durations of every pass of every timed step
    stage_ms = [[0.0] * 5 for _ in passes]
    for s in range(K):
        for n in range(len(passes)):
            e = evs[s][n]
            for j in range(5):
                stage_ms[n][j] += e[j].elapsed_time(e[j + 1]) / K
    region_s = ms / 1e3
    tf_peak, tf_name = tensor_peak(peaks, region_s)
    hbm = peaks["hbm_gbs"]

    def kernel_roof(kname, bytes_, flops, t_ms, launch):
        """Roofline entry of one kernel: its own bound (weight bytes at HBM peak against
        FLOPs at the bf16 peak), achieved = algorithmic work / mean launch time."""
        t_b = bytes_ / (hbm * 1e9)
        t_f = flops / (tf_peak * 1e12)
        if t_b >= t_f:
            a = bytes_ / (t_ms / 1e3) / 1e9
            return dict(bound="hbm", achieved=round(a, 1), peak=hbm, unit="GB/s", frac=round(a / hbm, 4),
                        kernel=kname, launch=launch, algorithmic_bytes_per_launch=int(bytes_),
                        us_per_launch=round(t_ms * 1e3, 2), peak_source=f"{peaks['source']} hbm_gbs")
        a = flops / (t_ms / 1e3) / 1e12
        return dict(bound="tensor", achieved=round(a, 1), peak=tf_peak, unit="TFLOP/s",
                    frac=round(a / tf_peak, 4), kernel=kname, launch=launch,
                    algorithmic_flops_per_launch=int(flops), us_per_launch=round(t_ms * 1e3, 2),
                    peak_source=f"{peaks['source']} {tf_name}")

    I2 = 2 * cfg.I
    blk_bytes = blk_flops = 0.0
    sweep_out = []
    gu_roofs, dn_roofs = [], []
    for n, p in enumerate(passes):
        T = p["T"]
        wb = 1 if spec.get("fp8") else 2   # bytes per expert weight (FP8: + a scale per row)
        b_gu = p["touched"] * I2 * (cfg.D * wb + (4 if wb == 1 else 0)) + (2 * cfg.I_s * cfg.D * 2 if cfg.I_s else 0)
        f_gu = 2.0 * T * cfg.k * I2 * cfg.D + (2.0 * T * 2 * cfg.I_s * cfg.D if cfg.I_s else 0)
        b_dn = p["touched"] * cfg.D * (cfg.I * wb + (4 if wb == 1 else 0)) + (cfg.I_s * cfg.D * 2 if cfg.I_s else 0)
        f_dn = 2.0 * T * cfg.k * cfg.I * cfg.D + (2.0 * T * cfg.I_s * cfg.D if cfg.I_s else 0)
        gu_roofs.append((b_gu, f_gu, stage_ms[n][2], T))
        dn_roofs.append((b_dn, f_dn, stage_ms[n][3], T))
        b = algorithmic_bytes(T, cfg.D, cfg.E, cfg.k, cfg.I, p["touched"], cfg.I_s, cfg.shared_gated,
                              residual=chain, fp8_experts=bool(spec.get("fp8")))
        f = algorithmic_flops(T, cfg.D, cfg.E, cfg.k, cfg.I, cfg.I_s, cfg.shared_gated)
        blk_bytes += b
        blk_flops += f
        if len(passes) > 1 and not chain:
            t_ms = per_T_ms[T]
            t_roof = max(b / (hbm * 1e9), f / (tf_peak * 1e12))
            entry = dict(
                T=T, path=p["path"], us=round(t_ms * 1e3, 2), tokens_per_s=round(T / (t_ms / 1e3), 1),
                roofline_us=round(t_roof * 1e6, 2), roofline_frac=round(t_roof / (t_ms / 1e3), 4),
                touched=p["touched"], max_load=p["max_load"])
            if p["path"] == "decode":   # one kernel: the whole block between the first two events
                entry["kernel_us_with_events"] = round(stage_ms[n][0] * 1e3, 2)
                entry["kernel_gbs"] = round(b / (stage_ms[n][0] / 1e3) / 1e9, 1)
            else:
                entry["stages_us_with_events"] = dict(zip(STAGES, [round(v * 1e3, 2) for v in stage_ms[n]]))
                entry["gate_up_gbs"] = round(b_gu / (stage_ms[n][2] / 1e3) / 1e9, 1)
                entry["down_gbs"] = round(b_dn / (stage_ms[n][3] / 1e3) / 1e9, 1)
            sweep_out.append(entry)

    def dominant(rs, kname):
        if chain:   # every layer has the same shape: average them
            b = sum(r[0] for r in rs) / len(rs)
            f = sum(r[1] for r in rs) / len(rs)
            t = sum(r[2] for r in rs) / len(rs)
            return kernel_roof(kname, b, f, t, f"T={rs[0][3]} (mean of {len(rs)} layers)")
        b, f, t, T = rs[-1]          # the largest pass: one launch shape, one ncu capture
        return kernel_roof(kname, b, f, t, f"T={T}")

    if passes[-1]["path"] == "decode":
        # one kernel for the whole block: its roofline is the block's bytes over its duration
        T = passes[-1]["T"]
        b = algorithmic_bytes(T, cfg.D, cfg.E, cfg.k, cfg.I, passes[-1]["touched"], cfg.I_s, cfg.shared_gated,
                              residual=chain, fp8_experts=bool(spec.get("fp8")))
        f = algorithmic_flops(T, cfg.D, cfg.E, cfg.k, cfg.I, cfg.I_s, cfg.shared_gated)
        roof = kernel_roof("decode_block_kernel", b, f, stage_ms[-1][0], f"T={T}")
        roof_dn = None
    else:
        roof = dominant(gu_roofs, "tc_gemm_kernel<gate_up>")
        roof_dn = dominant(dn_roofs, "tc_gemm_kernel<down>")
    tag = {"decode": "tc_gate_up_decode", "prefill": "tc_gemm_prefill"}.get(name, f"tc_gate_up_{name}")
    if passes[-1]["path"] == "decode":
        tag = "decode_block_t1_fp8" if spec.get("fp8") else "decode_block_t1"
    roof["traffic"] = profile_traffic(tag)
    blk_time = max(blk_bytes / (hbm * 1e9), blk_flops / (tf_peak * 1e12))
    res = dict(
        workload=describe(name, cfg, sweep, spec), tokens_per_step=tokens_per_step,
        value=round(agg["value"], 1), unit="tokens/s", ms_per_step=round(agg["ms_per_step"], 5),
        timing="CUDA graph replay" if use_graph else "eager",
        stage_timing=f"second timed replay of the {K} steps with stage events: {ms_events / K:.4f} ms/step",
        l2=("rotating %d weight copies (%.1f GB) > 126 MB L2" % (len(W), len(W) * weight_gb(cfg))
            if not chain else "48 distinct layers (%.1f GB) > 126 MB L2" % (48 * weight_gb(cfg))),
        roofline=roof, roofline_down=roof_dn,
        block_roofline=dict(time_us=round(blk_time * 1e6, 2), measured_us=round(agg["ms_per_step"] * 1e3, 2),
                            frac=round(blk_time / (agg["ms_per_step"] / 1e3), 4), bytes=int(blk_bytes),
                            flops=int(blk_flops), bound=("hbm" if blk_bytes / (hbm * 1e9) >=
                                                         blk_flops / (tf_peak * 1e12) else "tensor"),
                            peaks=f"hbm_gbs {hbm}, {tf_name} {tf_peak} ({peaks['source']})"),
        gpu_launches=int(sum(kernels_per_forward(p["T"], cfg.k, p["path"]) for p in passes) * K),
        clocks=sampler.summary())
    if not chain:
        res["stages_us_with_events"] = dict(zip(STAGES, [round(v * 1e3, 2) for v in stage_ms[-1]]))
        res["touched"], res["max_load"] = passes[-1]["touched"], passes[-1]["max_load"]
    else:
        res["stages_us_with_events"] = dict(zip(STAGES, [round(sum(stage_ms[n][j] for n in range(len(passes)))
                                                               / len(passes) * 1e3, 2) for j in range(5)]))
    if sweep_out:
        res["sweep"] = sweep_out

    # the router's balance loss and its gradient on this workload's own routing (prefill):
    # one moe_aux_loss call per step, CUDA events around a graph of K calls
    if name == "prefill":
        p = passes[-1]
        w = p["w"]
        logits, idx, _ = B.moe_route(p["x"], w["W_r"], cfg.k, cfg.norm_topk_prob, bias=w.get("bias"))
        aux_ws = torch.empty(int(B.load().moe_aux_loss_workspace_size(p["T"], cfg.E)), dtype=torch.uint8, device=device)
        for _ in range(3):
            B.moe_aux_loss(logits, idx, 0.001, ws=aux_ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream(device=device)):
            for _ in range(K):
                B.moe_aux_loss(logits, idx, 0.001, ws=aux_ws)
        g.replay()
        torch.cuda.synchronize()
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_ev.record()
        g.replay()
        b_ev.record()
        torch.cuda.synchronize()
        us = a_ev.elapsed_time(b_ev) * 1e3 / K
        # logits read twice (statistics, gradient), indices once, the gradient written once
        nbytes = 3 * p["T"] * cfg.E * 4 + p["T"] * cfg.k * 4
        res["aux_loss"] = dict(us_per_call=round(us, 2), kernels=3, algorithmic_bytes=nbytes,
                               achieved_gbs=round(nbytes / (us * 1e-6) / 1e9, 1),
                               hbm_frac=round(nbytes / (us * 1e-6) / 1e9 / hbm, 4),
                               note="loss and gradient of the Switch balance loss, T=%d, E=%d, k=%d" % (
                                   p["T"], cfg.E, cfg.k))
        del g
        # the backward pass for the same routing (all gradients: x, router weights, expert
        # weights, logits, routing weights), eager calls with CUDA events around K of them
        dy = inputs.upstream_grad(cfg, p["T"]).to(device)
        bw_dims = B.make_dims(p["T"], cfg.D, cfg.E, cfg.k, cfg.I, cfg.norm_topk_prob)
        bw_ws = torch.empty(int(B.load().moe_backward_workspace_size(ctypes.byref(bw_dims))), dtype=torch.uint8,
                            device=device)
        call = lambda: B.moe_backward(p["x"], w["W_r"], w["W_gate_up"], w["W_down"], dy, idx, cfg.norm_topk_prob,
                                      bias=w.get("bias"), ws=bw_ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        a_ev.record()
        for _ in range(K):
            call()
        b_ev.record()
        torch.cuda.synchronize()
        ms = a_ev.elapsed_time(b_ev) / K
        R = p["T"] * cfg.k
        flops = 16 * R * cfg.D * cfg.I + 4 * p["T"] * cfg.E * cfg.D   # seven GEMMs
        tf = flops / (ms * 1e-3) / 1e12
        res["backward"] = dict(ms_per_call=round(ms, 4), kernels=20, gemm_flops=flops, achieved_tflops=round(tf, 1),
                               frac_of_bf16=round(tf / peaks["bf16_tflops"], 4),
                               note="moe_backward, T=%d, E=%d, k=%d, I=%d: recompute g/u, z = W_down^T dy, "
                                    "dW_down, dX, dW_gate_up, dW_r, router dx (warp-MMA grouped GEMMs)" % (
                                        p["T"], cfg.E, cfg.k, cfg.I))
        del bw_ws

    # end to end through the public API with host buffers (eager, copies inside the region):
    # each pass's input goes up on one copy stream and its output comes back on another, and
    # consecutive steps alternate between two sets of device buffers, so copies overlap the
    # other passes' and the neighbouring steps' forwards, as a pipelining caller's do; events
    # order every buffer's reuse
    if with_e2e and not chain:
        hx = [p["x"].cpu().pin_memory() for p in passes]
        hy = [torch.empty(p["out"].shape, dtype=p["out"].dtype).pin_memory() for p in passes]
        NB = 2
        dx = [[torch.empty_like(p["x"]) for p in passes] for _ in range(NB)]
        dout = [[torch.empty_like(p["out"]) for p in passes] for _ in range(NB)]
        main = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
        in_ready = [[torch.cuda.Event() for _ in passes] for _ in range(NB)]
        fwd_done = [[torch.cuda.Event() for _ in passes] for _ in range(NB)]
        out_read = [[torch.cuda.Event() for _ in passes] for _ in range(NB)]

        def e2e_step(b):
            for n in range(len(passes)):
                with torch.cuda.stream(up):
                    up.wait_event(fwd_done[b][n])    # the forward that last read dx[b][n]
                    dx[b][n].copy_(hx[n], non_blocking=True)
                    in_ready[b][n].record(up)
            for n, p in enumerate(passes):
                main.wait_event(in_ready[b][n])
                main.wait_event(out_read[b][n])      # the last copy back of out[b][n] is done
                w = p["w"]
                B.moe_forward_ex(dx[b][n], w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, cfg.norm_topk_prob,
                                 out=dout[b][n], ws=p["ws"], opts=p["opts"])
                fwd_done[b][n].record(main)
                with torch.cuda.stream(down):
                    down.wait_event(fwd_done[b][n])
                    hy[n].copy_(dout[b][n], non_blocking=True)
                    out_read[b][n].record(down)

        for i in range(max(1, args.warmup)):
            e2e_step(i % NB)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(main)
        up.wait_event(s0)                            # no copy starts before the region
        for i in range(K):
            e2e_step(i % NB)
        for evs_b in out_read:                       # ... and the region ends after the last one
            for ev in evs_b:
                main.wait_event(ev)
        s1.record(main)
        torch.cuda.synchronize()
        e_ms = s0.elapsed_time(s1)
        if world > 1:
            t = torch.tensor([e_ms], device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        bytes_in = sum(p["x"].numel() * 2 for p in passes)
        res["e2e"] = dict(value=round(world * tokens_per_step * K / (e_ms / 1e3), 1), unit="tokens/s",
                          h2d_bytes_per_step=bytes_in, d2h_bytes_per_step=bytes_in,
                          timing="eager; copies on two copy streams and two buffer sets, overlapping "
                                 "other passes' and neighbouring steps' forwards")
    del passes, W, x0, evs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, cfg, L_cpu


# ------------------------------------------------------------------ CPU oracle legs

def oracle_sample_rate(cfg, x, w, rows, threads):
    """Oracle tokens/s over `rows` with `threads` threads (one forward per row)."""
    from oracle import oracle as O
    t0 = time.perf_counter()
    O.forward_rows(x, w["W_r"], w["W_gate_up"], w["W_down"], cfg.k, rows, norm=cfg.norm_topk_prob,
                   bias=w.get("bias"), shared_gate_up=w.get("shared_gate_up"),
                   shared_down=w.get("shared_down"), shared_gate=w.get("shared_gate"), threads=threads)
    return len(rows) / (time.perf_counter() - t0)


def cpu_baseline(cfg, L=None, target_cpu_s=4.0, layers=1):
    """The oracle as it stands on this host, on a bounded sample of the workload: on one core
    and on every core available to the process."""
    from oracle import oracle as O
    from sparse_fp32_softmax_b200 import inputs
    if L is None:
        L = inputs.make_layer(cfg, T=cfg.T)
    threads = O.cpu_threads_available()
    first = oracle_sample_rate(cfg, L["x"], L, [0], 1)            # tokens/s on one core (1 token)
    n1 = int(max(1, min(cfg.T, target_cpu_s / 2 * first)))
    one = oracle_sample_rate(cfg, L["x"], L, list(range(n1)), 1)
    n = int(max(threads, min(2048, target_cpu_s * one * threads / 2)))
    n = min(n, cfg.T)
    rate = oracle_sample_rate(cfg, L["x"], L, list(range(n)), threads)
    per = f", rate divided by {layers} layers" if layers > 1 else ""
    return dict(value=round(rate / layers, 3), unit="tokens/s", cores=threads, kind="oracle",
                sample=f"first {n} tokens of the T={cfg.T} batch, one FP64 block pass each, on {threads} "
                       f"cores{per}",
                single_core=dict(value=round(one / layers, 3), unit="tokens/s", cores=1,
                                 sample=f"first {n1} tokens, one core{per}"))


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
    ap.add_argument("--extra", default=DEFAULT_EXTRA,
                    help="comma-separated workloads measured after the headline one, or 'none'")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=None,
                    help="decode weight copies in rotation (default: one per pass of a step)")
    ap.add_argument("--sweep", default=None,
                    help="token counts of the headline workload's passes, e.g. 8 or 1,256 "
                         "(default: the workload's own; used to profile one size)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep:
        try:
            sw = tuple(int(t) for t in args.sweep.split(","))
        except ValueError:
            ap.error("--sweep takes comma-separated token counts")
        if not sw or min(sw) < 1:
            ap.error("--sweep takes positive token counts")
        WORKLOADS[args.workload] = dict(WORKLOADS[args.workload], sweep=sw)
    extra = [] if args.extra in ("", "none") else [w for w in args.extra.split(",") if w != args.workload]
    for w in extra:
        if w not in WORKLOADS:
            ap.error(f"unknown workload {w}")
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
    peaks = load_peaks()
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    res, cfg, L_cpu = measure(args.workload, args, rank, world, device, peaks, with_e2e=True)
    line = dict(
        metric=METRIC, value=res["value"], unit="tokens/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=res["ms_per_step"], higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16", data="synthetic",
        config=dict(workload=res["workload"], tokens_per_step=res["tokens_per_step"], l2=res["l2"],
                    timing=res["timing"], stage_timing=res["stage_timing"],
                    parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        roofline=res["roofline"], roofline_down=res["roofline_down"], block_roofline=res["block_roofline"],
        gpu_launches=res["gpu_launches"], clocks=res["clocks"], e2e=res.get("e2e"),
        stages_us_with_events=res["stages_us_with_events"])
    if "sweep" in res:
        line["sweep"] = res["sweep"]
    if "aux_loss" in res:
        line["aux_loss"] = res["aux_loss"]
    if "backward" in res:
        line["backward"] = res["backward"]
    if want_cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, L_cpu, layers=WORKLOADS[args.workload]["layers"])
    del L_cpu
    if extra:
        line["workloads"] = {}
        keras_cpu = None
        for wname in extra:
            r, c, Lc = measure(wname, args, rank, world, device, peaks, with_e2e=False)
            if want_cpu:
                if WORKLOADS[wname]["layers"] > 1:
                    if keras_cpu is None:
                        keras_cpu = cpu_baseline(c, None)
                    nl = WORKLOADS[wname]["layers"]
                    cb = dict(keras_cpu)
                    cb["value"] = round(keras_cpu["value"] / nl, 3)
                    cb["sample"] = keras_cpu["sample"] + f", rate divided by {nl} layers"
                    cb["single_core"] = dict(keras_cpu["single_core"])
                    cb["single_core"]["value"] = round(keras_cpu["single_core"]["value"] / nl, 3)
                    r["cpu_baseline"] = cb
                else:
                    r["cpu_baseline"] = cpu_baseline(c, Lc)
                    if wname == "keras":
                        keras_cpu = r["cpu_baseline"]
            line["workloads"][wname] = r
            del Lc
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
