"""Seeded synthetic inputs for the MoE FFN block.

This module holds no step of the method: it only draws tensors.  Both the CUDA path's tests
and benchmark and the CPU oracle's tests take their inputs from here.

Recipe (the workloads of the block's five standard configurations):
  * bf16 values are FP32 draws from a seeded ``torch.Generator`` rounded to bf16
    (round-to-nearest-even, torch's ``.to(torch.bfloat16)``);
  * x ~ N(0, 1); W_r, W_gate_up, W_down and the shared expert's tensors ~ N(0, 0.02);
  * the seed of tensor ``tid`` of a configuration with seed ``s`` is ``1000*s + tid``; layer l
    of the 48-block chain uses seed ``1000*s + 100 + l`` as its base;
  * "tiny" gives four token rows exactly tied top logits: those rows are one-hot (or zero)
    so that each logit equals one router weight exactly, under any summation order;
  * "zipf" adds an FP32 router bias b[e] = -1.1 * ln(r[e]) with r a seeded permutation of
    1..E, which makes the prior expert popularity Zipf(1.1).
Weights use the stacked layouts gate_up [E, 2I, D] (gate rows first) and down [E, D, I].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

# tensor ids inside a configuration's seed space
TID_X, TID_WR, TID_WGU, TID_WDN, TID_SGU, TID_SDN, TID_SG, TID_BIAS = range(8)
TID_DY = 8   # the upstream gradient dy of the backward pass


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    D: int
    E: int
    k: int
    I: int
    norm_topk_prob: bool
    seed: int
    I_s: int = 0                 # shared expert width (0 = no shared expert)
    shared_gated: bool = False
    zipf_s: float | None = None  # router bias exponent
    tie_rows: tuple = ()
    chain_layers: int = 0        # >0: a chain of residual MoE blocks
    T_sweep: tuple = ()
    x_pool_rows: int = 0         # decode: x = first T rows of one [x_pool_rows, D] draw
    notes: str = ""


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, D=256, E=8, k=2, I=128, norm_topk_prob=True, seed=0,
                      tie_rows=(5, 21, 42, 63)),
    "decode": MoEConfig("decode", T=256, D=2048, E=128, k=8, I=768, norm_topk_prob=True, seed=1,
                        T_sweep=(1, 8, 32, 128, 256), x_pool_rows=256),
    "prefill": MoEConfig("prefill", T=8192, D=2048, E=128, k=8, I=768, norm_topk_prob=True, seed=2,
                         notes="8 x (900 image-like + 124 text-like) rows, all N(0,1)"),
    "keras": MoEConfig("keras", T=4096, D=2048, E=60, k=4, I=1408, norm_topk_prob=True, seed=3,
                       chain_layers=48),
    "zipf": MoEConfig("zipf", T=4096, D=2048, E=512, k=10, I=512, norm_topk_prob=True, seed=4,
                      I_s=512, shared_gated=True, zipf_s=1.1),
}

# Tie rows of "tiny": token row -> (one-hot column j or None for a zero row,
# {expert: logit value}, expected experts in slot order).  All values are exact in bf16.
TINY_TIES = {
    5: (0, {3: 0.0625, 6: 0.0625}, (3, 6)),                       # two-way tie at the top
    21: (1, {5: 0.09375, 2: 0.03125, 7: 0.03125}, (5, 2)),        # clear top, tie for 2nd
    42: (2, {1: 0.046875, 4: 0.046875, 6: 0.046875}, (1, 4)),     # three-way tie at the top
    63: (None, {}, (0, 1)),                                       # zero row: all tied
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu", gen_device="cpu") -> torch.Tensor:
    """FP32 N(0, std) draw from a seeded generator, rounded to bf16."""
    g = _gen(seed, gen_device)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=gen_device)
    if std != 1.0:
        t.mul_(std)
    t = t.to(torch.bfloat16)
    return t.to(device) if str(device) != str(gen_device) else t


def zipf_bias(E: int, s: float, seed: int) -> torch.Tensor:
    """b[e] = -s * ln(r[e]), r a seeded permutation of 1..E (FP32)."""
    r = torch.randperm(E, generator=_gen(seed)).to(torch.float64) + 1.0
    return (-s * torch.log(r)).to(torch.float32)


def _apply_tiny_ties(x: torch.Tensor, W_r: torch.Tensor, E: int) -> None:
    for row, (col, vals, _) in TINY_TIES.items():
        x[row].zero_()
        if col is None:
            continue
        x[row, col] = 1.0
        # the whole router column j is rewritten: distinct values below every tie value
        W_r[:, col] = torch.tensor([-0.01 * (e + 1) for e in range(E)], dtype=torch.float32).to(torch.bfloat16)
        for e, v in vals.items():
            W_r[e, col] = v


def make_layer(cfg: MoEConfig, T: int | None = None, layer: int | None = None, device="cpu",
               gen_device="cpu", with_x: bool = True) -> dict:
    """All tensors of one block of ``cfg`` (x for T tokens).

    ``layer`` selects a block of the residual chain (its own weight seeds).  ``gen_device``
    "cuda" draws from torch's CUDA generator instead (used only for chain layers that no
    oracle test replays).
    """
    T = cfg.T if T is None else int(T)
    base = 1000 * cfg.seed if layer is None else 1000 * cfg.seed + 100 + int(layer)
    D, E, I = cfg.D, cfg.E, cfg.I
    kw = dict(device=device, gen_device=gen_device)
    out = {}
    if with_x:
        if cfg.x_pool_rows:
            pool = normal_bf16((cfg.x_pool_rows, D), 1.0, 1000 * cfg.seed + TID_X, **kw)
            out["x"] = pool[:T].contiguous()
        else:
            out["x"] = normal_bf16((T, D), 1.0, 1000 * cfg.seed + TID_X, **kw)
    out["W_r"] = normal_bf16((E, D), 0.02, base + TID_WR, **kw)
    out["W_gate_up"] = normal_bf16((E, 2 * I, D), 0.02, base + TID_WGU, **kw)
    out["W_down"] = normal_bf16((E, D, I), 0.02, base + TID_WDN, **kw)
    out["bias"] = None
    if cfg.zipf_s is not None:
        out["bias"] = zipf_bias(E, cfg.zipf_s, base + TID_BIAS).to(device)
    out["shared_gate_up"] = out["shared_down"] = out["shared_gate"] = None
    if cfg.I_s:
        out["shared_gate_up"] = normal_bf16((2 * cfg.I_s, D), 0.02, base + TID_SGU, **kw)
        out["shared_down"] = normal_bf16((D, cfg.I_s), 0.02, base + TID_SDN, **kw)
        if cfg.shared_gated:
            out["shared_gate"] = normal_bf16((D,), 0.02, base + TID_SG, **kw)
    if cfg.tie_rows and with_x:
        x, W_r = out["x"].cpu(), out["W_r"].cpu()
        _apply_tiny_ties(x, W_r, E)
        out["x"], out["W_r"] = x.to(device), W_r.to(device)
    return out


def upstream_grad(cfg: MoEConfig, T: int | None = None, device="cpu") -> torch.Tensor:
    """dy [T, D] for the backward pass: N(0, 1) rounded to bf16, seeded per configuration."""
    T = cfg.T if T is None else int(T)
    return normal_bf16((T, cfg.D), 1.0, 1000 * cfg.seed + TID_DY, device=device)


def coverage_rows(T: int, n_random: int, seed: int, extra=()) -> list:
    """A sorted sample of token rows: ``n_random`` seeded random rows, the first and last
    rows, and any ``extra`` rows (e.g. segment boundaries of a permutation)."""
    g = _gen(seed + 7919)
    n_random = min(n_random, T)
    rnd = torch.randperm(T, generator=g)[:n_random].tolist()
    rows = set(rnd) | {0, T - 1} | {int(r) for r in extra if 0 <= int(r) < T}
    return sorted(rows)
