"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Stage-wise (router, permutation) and end to end (the whole block) on the standard
workloads, and the edge cases: T = 1, ragged T, k = 1, k = E, E = 1, norm_topk_prob off,
all tokens on one expert, zero input, E = 512 with k = 16.  The 48-block residual chain is
in test_gpu_chain.py, failure detection in test_gpu_failure.py.
"""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import (W_ATOL, assert_block_output, assert_y_close, check_routing,
                               logit_deltas)

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, O.cpu_threads_available()))


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()
    O.build()


_layers = {}


def layer(name, T=None):
    key = (name, T)
    if key not in _layers:
        cfg = inputs.CONFIGS[name]
        L = inputs.make_layer(cfg, T=T)
        _layers[key] = (cfg, L, {k: (v.cuda() if v is not None else None) for k, v in L.items()})
    return _layers[key]


def to_f64(y):
    return y.double().numpy()


def run_forward(cfg, G, path="auto", x=None, residual=None, k=None, norm=None):
    x = G["x"] if x is None else x
    k = cfg.k if k is None else k
    norm = cfg.norm_topk_prob if norm is None else norm
    T, E = x.shape[0], G["W_r"].shape[0]
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    y32 = torch.empty(x.shape, dtype=torch.float32, device="cuda")
    out = B.moe_forward_ex(x, G["W_r"], G["W_gate_up"], G["W_down"], k, norm,
                           router_bias=G.get("bias"), shared_gate_up=G.get("shared_gate_up"),
                           shared_down=G.get("shared_down"), shared_gate=G.get("shared_gate"),
                           residual=residual, logits_out=logits, topk_idx_out=idx, topk_w_out=w,
                           path=path, out_f32=y32)
    torch.cuda.synchronize()
    run_forward.last_f32 = y32.cpu()
    return out.cpu(), idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()


def compare_block(cfg, L, G, rows, path="auto", x_cpu=None, residual_cpu=None, k=None, norm=None,
                  what=""):
    """Run the block on the GPU, check routing of `rows` and y against the oracle."""
    k = cfg.k if k is None else k
    norm = cfg.norm_topk_prob if norm is None else norm
    x_cpu = L["x"] if x_cpu is None else x_cpu
    res_gpu = residual_cpu.cuda() if residual_cpu is not None else None
    y, idx, w, logits = run_forward(cfg, G, path=path, x=x_cpu.cuda(), residual=res_gpu, k=k, norm=norm)
    y32 = run_forward.last_f32
    rows = np.asarray(sorted(set(int(r) for r in rows)), np.int32)
    # selection from the GPU's own logits is bit-exact; weights within 1e-6
    o_idx, o_w = O.select(logits, k, norm)
    assert np.array_equal(o_idx, idx), what
    assert np.abs(o_w - w).max() <= W_ATOL, what
    # against the FP64 oracle: exact on decisive tokens, valid elsewhere
    y_o, oi, ow, ol = O.forward_rows(x_cpu, L["W_r"], L["W_gate_up"], L["W_down"], k, rows, norm=norm,
                                     bias=L.get("bias"), shared_gate_up=L.get("shared_gate_up"),
                                     shared_down=L.get("shared_down"),
                                     shared_gate=L.get("shared_gate"), residual=residual_cpu,
                                     threads=THREADS)
    delta = logit_deltas(x_cpu[torch.from_numpy(rows).long()], L["W_r"], ol)
    assert (np.abs(logits[rows] - ol) <= delta + 1e-30).all(), what
    nd, nother = check_routing(idx[rows], oi, ol, delta, k)
    # y: where the GPU routed differently (only possible on non-decisive tokens) the
    # reference is the oracle's combine under the GPU's (valid) routing
    y_ref = y_o.copy()
    diff_rows = [n for n, t in enumerate(rows) if idx[t].tolist() != oi[n].tolist()]
    if diff_rows:
        sub = rows[diff_rows]
        y_ref[diff_rows] = O.combine_rows(x_cpu, idx, w, sub, L["W_gate_up"], L["W_down"],
                                          shared_gate_up=L.get("shared_gate_up"),
                                          shared_down=L.get("shared_down"),
                                          shared_gate=L.get("shared_gate"),
                                          residual=residual_cpu, threads=THREADS)
    sel = torch.from_numpy(rows).long()
    rel, mx = assert_block_output(y[sel], y32[sel], y_ref, what)
    return dict(rel_l2=rel, max_abs_over_rms=mx, decisive=nd, other=nother, idx=idx, y=y)


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("repeat", [1, 3])   # T = 64 (CUDA-core router), 192 (tcgen05 router)
def test_route_tiny_ties(repeat):
    cfg, L, G = layer("tiny")
    x = G["x"].repeat(repeat, 1).contiguous()
    logits, idx, w = B.moe_route(x, G["W_r"], cfg.k, cfg.norm_topk_prob)
    torch.cuda.synchronize()
    idx, w, logits = idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()
    for rep in range(repeat):
        for row, (_, _, expect) in inputs.TINY_TIES.items():
            t = rep * cfg.T + row
            assert tuple(idx[t].tolist()) == expect, (t, idx[t])
        for row in (5, 42, 63):
            assert (w[rep * cfg.T + row] == 0.5).all()
    o_idx, o_w = O.select(logits, cfg.k, True)
    assert np.array_equal(o_idx, idx)
    assert np.abs(o_w - w).max() <= W_ATOL


@pytest.mark.parametrize("name,T", [("decode", 1), ("decode", 256), ("prefill", None),
                                    ("keras", None), ("zipf", None)])
def test_route_stagewise(name, T):
    cfg, L, G = layer(name, T)
    x = G["x"]
    logits, idx, w = B.moe_route(x, G["W_r"], cfg.k, cfg.norm_topk_prob, bias=G.get("bias"))
    torch.cuda.synchronize()
    idx, w, logits = idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()
    o_idx, o_w = O.select(logits, cfg.k, cfg.norm_topk_prob)
    assert np.array_equal(o_idx, idx)                 # every token, bit-exact
    assert np.abs(o_w - w).max() <= W_ATOL
    Tn = x.shape[0]
    rows = np.asarray(inputs.coverage_rows(Tn, 512, cfg.seed), np.int32)
    ol = O.router_logits(L["x"][torch.from_numpy(rows).long()], L["W_r"], L.get("bias"))
    delta = logit_deltas(L["x"][torch.from_numpy(rows).long()], L["W_r"], ol)
    assert (np.abs(logits[rows] - ol) <= delta).all()
    oi, _ = O.select(ol, cfg.k, cfg.norm_topk_prob)
    nd, no = check_routing(idx[rows], oi, ol, delta, cfg.k)
    # the FP32 bound is rigorous and loose: most tokens are still decisive
    assert nd >= 0.4 * len(rows), (nd, no)


# ------------------------------------------------------------------ permute

@pytest.mark.parametrize("tile_m", [1, 8, 128])
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (37, 3, 9), (300, 8, 128), (5000, 10, 512)])
def test_permute_bit_exact(tile_m, T, k, E):
    g = torch.Generator().manual_seed(T * 7 + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    w = torch.rand(T, k, generator=g)
    x = torch.randn(T, 128, generator=g).to(torch.bfloat16)
    out = B.moe_permute(idx.cuda(), E, tile_m, topk_w=w.cuda(), x=x.cuda(), want_x_perm=True)
    torch.cuda.synchronize()
    counts, offsets, row_token, slot_row = O.permute(idx.numpy(), E, tile_m)
    assert np.array_equal(out["counts"].cpu().numpy(), counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), offsets)
    rt = out["row_token"].cpu().numpy()
    assert np.array_equal(rt, row_token)
    assert np.array_equal(out["slot_row"].cpu().numpy(), slot_row)
    rw = out["row_weight"].cpu().numpy()
    flat_w = w.numpy().reshape(-1)
    assert np.array_equal(rw[slot_row], flat_w)
    assert (rw[rt < 0] == 0).all()
    xp = out["x_perm"].cpu()
    valid = torch.from_numpy(rt >= 0)
    assert torch.equal(xp[valid], x[torch.from_numpy(rt[rt >= 0]).long()])
    assert (xp[~valid] == 0).all()


# ------------------------------------------------------------------ whole block

def test_forward_tiny():
    cfg, L, G = layer("tiny")
    r = compare_block(cfg, L, G, range(cfg.T), what="tiny")
    for row, (_, _, expect) in inputs.TINY_TIES.items():
        assert tuple(r["idx"][row].tolist()) == expect
    assert (r["y"][63] == 0).all()


@pytest.mark.parametrize("T", [1, 8, 32, 128, 256])
def test_forward_decode_sweep(T):
    cfg, L, G = layer("decode", T)
    compare_block(cfg, L, G, range(T), what=f"decode T={T}")


def _boundary_rows(cfg, L, n_random=256):
    """Coverage rows: seeded random rows plus, from the oracle's own routing of every token,
    the first and last rows of each expert segment and of each token tile."""
    ol = O.router_logits(L["x"], L["W_r"], L.get("bias"))
    oi, _ = O.select(ol, cfg.k, cfg.norm_topk_prob)
    counts, offsets, row_token, _ = O.permute(oi, cfg.E, 1)
    extra = []
    for e in range(cfg.E):
        c, o = int(counts[e]), int(offsets[e])
        for tile in (128, 256):
            for s in range(0, c, tile):
                extra += [row_token[o + s], row_token[o + min(c, s + tile) - 1]]
    rows = inputs.coverage_rows(L["x"].shape[0], n_random, cfg.seed, extra)
    return rows, counts


@pytest.mark.parametrize("name", ["prefill", "keras", "zipf"])
def test_forward_large_configs(name):
    cfg, L, G = layer(name)
    rows, counts = _boundary_rows(cfg, L)
    r = compare_block(cfg, L, G, rows, what=name)
    print(f"{name}: rows={len(rows)} rel_l2={r['rel_l2']:.2e} max/rms={r['max_abs_over_rms']:.2e} "
          f"decisive={r['decisive']} other={r['other']} max_load={counts.max()} mean_load={counts.mean():.1f}")


def _small_layer(T, D=256, E=16, k=4, I=256, seed=5, I_s=0, bias=None):
    cfg = inputs.MoEConfig("edge", T=T, D=D, E=E, k=k, I=I, norm_topk_prob=True, seed=seed, I_s=I_s,
                           shared_gated=bool(I_s))
    L = inputs.make_layer(cfg)
    if bias is not None:
        L["bias"] = bias
    G = {k_: (v.cuda() if v is not None else None) for k_, v in L.items()}
    return cfg, L, G


@pytest.mark.parametrize("T", [1, 7, 65, 129, 300])
def test_forward_ragged_T(T):
    cfg, L, G = _small_layer(T)
    compare_block(cfg, L, G, range(T), what=f"ragged T={T}")


@pytest.mark.parametrize("E,k,norm", [(16, 1, True), (8, 8, True), (16, 4, False), (1, 1, True),
                                      (512, 16, True)])
def test_forward_k_E_norm(E, k, norm):
    cfg, L, G = _small_layer(96, E=E, k=k)
    compare_block(cfg, L, G, range(96), k=k, norm=norm, what=f"E={E} k={k} norm={norm}")


def test_forward_all_tokens_one_expert():
    bias = torch.zeros(16)
    bias[3] = 100.0
    cfg, L, G = _small_layer(600, bias=bias)
    r = compare_block(cfg, L, G, range(0, 600, 3), what="skewed")
    assert (r["idx"][:, 0] == 3).all()


def test_forward_shared_expert_and_residual():
    cfg, L, G = _small_layer(200, I_s=384)
    res = torch.randn(200, 256, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    compare_block(cfg, L, G, range(200), residual_cpu=res, what="shared+res")
    # ungated shared expert
    L2 = dict(L, shared_gate=None)
    G2 = dict(G, shared_gate=None)
    compare_block(cfg, L2, G2, range(200), what="ungated")


def test_forward_single_sm_wide_tiles(monkeypatch):
    """The one-CTA wide tiles (used where SM pairs cannot be scheduled) on a wide shape: the
    interleaved gate_up and the wide down, against the oracle."""
    monkeypatch.setenv("MOE_B200_NO_PAIRS", "1")
    cfg, L, G = _small_layer(600, E=8, k=4)
    compare_block(cfg, L, G, range(600), path="grouped", what="single-SM wide tiles")


@pytest.mark.parametrize("T", [5, 300])
def test_forward_dims_not_multiple_of_256(T):
    """D = I = 384: gate_up K and feature tiles of 128 (pair tiles at T = 300), down rows not a
    multiple of 256 (the one-CTA wide down tiles at T = 300, narrow tiles at T = 5)."""
    cfg, L, G = _small_layer(T, D=384, E=16, k=4, I=384)
    compare_block(cfg, L, G, range(T), path="grouped", what=f"D=I=384 T={T}")


@pytest.mark.parametrize("T", [2, 5, 9])
def test_forward_split_tail_with_shared_expert(T):
    """Decode-sized batches whose expert GEMMs split their last items along K (a few dozen
    items on 148 SMs): gate_up over D = 512 (8 K stages, split 3 or 4 ways: uneven slices),
    down over I = 256 and the shared expert's I_s = 128 (the split is bounded by the shared
    segment's 2 K stages), with the gated shared expert and a residual."""
    cfg, L, G = _small_layer(T, D=512, E=64, k=4, I=256, I_s=128)
    res = torch.randn(T, 512, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    compare_block(cfg, L, G, range(T), path="grouped", residual_cpu=res, what=f"split tail T={T}")


def test_forward_zero_input():
    cfg, L, G = _small_layer(40)
    x0 = torch.zeros_like(L["x"])
    res = torch.randn(40, 256, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    y, idx, w, _ = run_forward(cfg, G, x=x0.cuda(), residual=res.cuda())
    assert torch.equal(y, res)                                 # block(0) = 0 exactly
    assert (idx == np.arange(cfg.k)[None, :]).all()           # all logits 0 -> lowest indices
    assert np.abs(w - 1.0 / cfg.k).max() <= W_ATOL


def test_determinism_and_batch_invariance():
    """Bitwise-equal reruns of the same batch.  A token's routing (experts and FP32 weights)
    does not depend on the other tokens of the batch within a router kernel's range (T <= 64
    runs the CUDA-core router, larger T the tensor-core one with a K split fixed by the shapes;
    the two sum the logits in different FP32 orders).  Its output agrees within the output
    tolerance: the expert GEMMs split the last wave's items along K, and how many items there
    are depends on the batch, so the FP32 summation order of y can change with it."""
    cfg, L, G = _small_layer(256)
    y1, i1, w1, l1 = run_forward(cfg, G)
    y2, i2, w2, l2 = run_forward(cfg, G)
    assert torch.equal(y1, y2) and (i1 == i2).all() and (w1 == w2).all() and (l1 == l2).all()
    y100, i100, w100, l100 = run_forward(cfg, G, x=G["x"][:100].contiguous())
    assert (l100 == l1[:100]).all() and (i100 == i1[:100]).all() and (w100 == w1[:100]).all()
    assert_y_close(to_f64(y100), to_f64(y1[:100]), "T=100 vs the first 100 of T=256")
    y64, i64, w64, l64 = run_forward(cfg, G, x=G["x"][:64].contiguous())
    y8, i8, w8, l8 = run_forward(cfg, G, x=G["x"][:8].contiguous())
    assert (l8 == l64[:8]).all() and (i8 == i64[:8]).all() and (w8 == w64[:8]).all()
    assert_y_close(to_f64(y8), to_f64(y64[:8]), "T=8 vs the first 8 of T=64")


def test_status_ok_after_a_forward():
    cfg, L, G = layer("decode", 128)
    dims = B.make_dims(128, cfg.D, cfg.E, cfg.k, cfg.I)
    ws = B.workspace(dims)
    B.moe_forward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK


def test_gpu_errors_before_launch():
    cfg, L, G = _small_layer(16)
    dims = B.make_dims(16, 256, 16, 4, 256)
    small = torch.empty(B.moe_workspace_size(dims) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_forward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], 4, ws=small)
    assert ei.value.status == B.MOE_ERR_WORKSPACE
    with pytest.raises(B.MoeError) as ei:
        B.moe_forward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], 17)
    assert ei.value.status == B.MOE_ERR_UNSUPPORTED


# ------------------------------------------------------------------ permutation at the
# workloads' own routing (the forward's internal tables and moe_permute)

@pytest.mark.parametrize("name,T", [("decode", 8), ("decode", 256), ("prefill", None), ("keras", None),
                                    ("zipf", None)])
def test_permutation_at_workload_routing(name, T):
    """The expert-sorted layout the forward builds from its own routing (per-expert counts and
    the row of every assignment, read back through expert_counts_out / slot_row_out), and
    moe_permute on the same routing with tile_m = 128, both bit-exact against the oracle's
    stable counting sort.  zipf's routing is heavily skewed (one expert takes almost every
    token, across many 4096-assignment chunks of the multi-block permutation)."""
    cfg, L, G = layer(name, T)
    x = G["x"]
    Tn = x.shape[0]
    idx = torch.empty(Tn, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(Tn, cfg.k, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.E, dtype=torch.int32, device="cuda")
    slot_row = torch.empty(Tn, cfg.k, dtype=torch.int32, device="cuda")
    B.moe_forward_ex(x, G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, cfg.norm_topk_prob,
                     router_bias=G.get("bias"), shared_gate_up=G.get("shared_gate_up"),
                     shared_down=G.get("shared_down"), shared_gate=G.get("shared_gate"),
                     topk_idx_out=idx, topk_w_out=w, expert_counts_out=counts, slot_row_out=slot_row)
    torch.cuda.synchronize()
    idx_h = idx.cpu().numpy()
    o_counts, o_offsets, o_row_token, o_slot_row = O.permute(idx_h, cfg.E, 1)
    assert np.array_equal(counts.cpu().numpy(), o_counts)
    assert np.array_equal(slot_row.cpu().numpy().reshape(-1), o_slot_row)
    # moe_permute on the same routing, tile-padded
    out = B.moe_permute(idx, cfg.E, 128, topk_w=w, x=x, want_x_perm=True)
    torch.cuda.synchronize()
    c, off, rt, sr = O.permute(idx_h, cfg.E, 128)
    assert np.array_equal(out["counts"].cpu().numpy(), c)
    assert np.array_equal(out["offsets"].cpu().numpy(), off)
    assert np.array_equal(out["row_token"].cpu().numpy(), rt)
    assert np.array_equal(out["slot_row"].cpu().numpy(), sr)
    rw = out["row_weight"].cpu().numpy()
    assert np.array_equal(rw[sr], w.cpu().numpy().reshape(-1))
    xp = out["x_perm"].cpu()
    valid = torch.from_numpy(rt >= 0)
    assert torch.equal(xp[valid], L["x"][torch.from_numpy(rt[rt >= 0]).long()])
    assert (xp[~valid] == 0).all()
    print(f"{name}: T={Tn} assignments={Tn * cfg.k} touched={(o_counts > 0).sum()} "
          f"max_load={o_counts.max()} chunks={(Tn * cfg.k + 4095) // 4096}")
