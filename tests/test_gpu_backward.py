"""moe_backward on the GPU against the oracle's FP64 backward (the same routing on both
sides, made by the oracle's router and selection from the seeded layer; dy from the seeded
upstream-gradient generator).

Tolerances, from the arithmetic: the GPU rounds the GEMM operands it computes (h, dg/du,
w dy, dlogits) to bf16 once (a relative error of at most 2^-9, about 2^-9/sqrt(3) rms) and
accumulates in FP32; the weights, x and dy are exact bf16 inputs.  A gradient that sums
products with one rounded operand then has a relative L2 error near 1.1e-3 (independent
roundings), so each tensor is checked to relative L2 <= 5e-3 and max-abs <= 1e-2 of its
largest entry.  dw and dlogits use only FP32 arithmetic on exact operands: 1e-4.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.test_gpu_parity import layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()
    O.build()


def close(name, got, ref, rel=5e-3, mx=1e-2):
    got = got.detach().cpu().double().numpy() if torch.is_tensor(got) else got
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    l2 = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert l2 <= rel and err.max() <= mx * max(scale, 1e-300), (name, l2, err.max(), scale)
    return l2


def run_case(name, T=None, residual=False, dl_add=False, rows=None, experts=None):
    cfg, L, G = layer(name, T)
    T = G["x"].shape[0]
    dy = inputs.upstream_grad(cfg, T)
    _, idx, _ = O.route(L["x"], L["W_r"], cfg.k, cfg.norm_topk_prob, bias=L.get("bias"))
    add = None
    if dl_add:   # the balance loss's gradient, as a trainer would add it
        _, add = O.aux_loss(O.router_logits(L["x"], L["W_r"], L.get("bias")), idx, 0.01)
        add = add.astype(np.float32)
    out = B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy.cuda(), torch.from_numpy(idx).cuda(),
                         cfg.norm_topk_prob, bias=G.get("bias"), residual=residual, with_dbias=True,
                         dlogits_add=None if add is None else torch.from_numpy(add).cuda())
    torch.cuda.synchronize()
    if experts is None:
        counts = np.bincount(idx.reshape(-1), minlength=cfg.E)
        experts = sorted({int(np.argmax(counts)), int(np.argmin(counts)), 0})
    sel = np.arange(T) if rows is None else np.asarray(rows)
    ref = O.backward(L["x"][sel], L["W_r"], L["W_gate_up"], L["W_down"], dy[sel], idx[sel], norm=cfg.norm_topk_prob,
                     bias=L.get("bias"), residual=residual, dlogits_add=None if add is None else add[sel],
                     experts=experts if rows is None else ())
    close("dx", out["dx"][sel], ref["dx"])
    close("dlogits", out["dlogits"][sel], ref["dlogits"], 1e-4, 1e-4)
    close("dw", out["dw"][sel], ref["dw"], 1e-4, 1e-4)
    if rows is None:   # sums over all tokens
        close("dW_r", out["dW_r"], ref["dW_r"])
        close("dbias", out["dbias"], ref["db"])
        close("dW_gate_up", out["dW_gate_up"][experts], ref["dW_gu"])
        close("dW_down", out["dW_down"][experts], ref["dW_dn"])
        unused = sorted(set(range(cfg.E)) - set(idx.reshape(-1).tolist()))
        for e in unused:
            assert not out["dW_gate_up"][e].any() and not out["dW_down"][e].any()
    return out


def test_backward_tiny_all_experts():
    """tiny: T=64, D=256, E=8, k=2, I=128, tie rows; every expert's weight gradients."""
    run_case("tiny", experts=list(range(8)))


def test_backward_many_rows_per_expert_residual_and_balance_loss():
    """tiny weights with T=1024: ~256 rows per expert (several 128-row tiles and 32-row K
    steps, ragged tails), a residual block, and the balance loss's logit gradient added."""
    run_case("tiny", T=1024, residual=True, dl_add=True, experts=list(range(8)))


def test_backward_workload_shape():
    """D=2048, E=128, k=8, I=768 (the decode / prefill layer) with 64 tokens: most experts get
    0-8 rows; the busiest, the idlest and expert 0 are checked in full."""
    run_case("decode", T=64)


def test_backward_zipf_bias():
    """E=512, k=10, I=512 with the Zipf router bias (its gradient is dbias), 48 tokens."""
    run_case("zipf", T=48)


def test_backward_prefill_sampled_tokens():
    """The prefill layer at full size (T=8192): dx, dlogits, dw of sampled tokens against the
    oracle run on those tokens alone (a token's input and logit gradients depend only on it)."""
    rows = inputs.coverage_rows(8192, 14, seed=5)
    run_case("prefill", rows=rows)


def test_backward_deterministic_and_norm_off():
    cfg, L, G = layer("tiny", 256)
    dy = inputs.upstream_grad(cfg, 256).cuda()
    _, idx, _ = O.route(L["x"], L["W_r"], cfg.k, False)
    idx = torch.from_numpy(idx).cuda()
    a = B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy, idx, False)
    b = B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy, idx, False)
    torch.cuda.synchronize()
    for key in a:
        if a[key] is not None:
            assert torch.equal(a[key], b[key]), key
    ref = O.backward(L["x"], L["W_r"], L["W_gate_up"], L["W_down"], dy.cpu(), idx.cpu(), norm=False)
    close("dx", a["dx"], ref["dx"])
    close("dlogits", a["dlogits"], ref["dlogits"], 1e-4, 1e-4)


def test_backward_bad_index_is_reported():
    """An expert index outside [0, E) is skipped and recorded: moe_get_device_status returns
    MOE_ERR_INVALID_ARG, and the call leaves the context usable."""
    cfg, L, G = layer("tiny")
    dy = inputs.upstream_grad(cfg).cuda()
    _, idx, _ = O.route(L["x"], L["W_r"], cfg.k, True)
    idx[3, 1] = cfg.E + 5
    lib = B.load()
    dims = B.make_dims(64, cfg.D, cfg.E, cfg.k, cfg.I, True)
    ws = torch.empty(int(lib.moe_backward_workspace_size(__import__("ctypes").byref(dims))), dtype=torch.uint8,
                     device="cuda")
    B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy, torch.from_numpy(idx).cuda(), True, ws=ws)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(ws) == B.MOE_ERR_INVALID_ARG
    assert torch.ones(4, device="cuda").sum().item() == 4.0


def test_backward_keras_shape_unpadded_E():
    """E=60 (not a multiple of 8: the logit-gradient operand is zero-padded to 64 columns and
    W_r's rows beyond 60 are not read), k=4, I=1408 (22 tiles of 2I), 40 tokens."""
    run_case("keras", T=40)


@pytest.mark.parametrize("T", [1, 3])
def test_backward_one_and_three_tokens(T):
    """T=1 and a ragged T=3 at the D=2048, E=128, k=8, I=768 layer: one row per chosen expert."""
    run_case("decode", T=T)


def test_backward_captured_in_a_cuda_graph():
    """moe_backward allocates and synchronises nothing, so it can be captured in a CUDA graph
    (after one eager call on the same shape); the replay is bitwise equal to the eager call."""
    cfg, L, G = layer("tiny", 1024)
    dy = inputs.upstream_grad(cfg, 1024).cuda()
    _, idx, _ = O.route(L["x"], L["W_r"], cfg.k, True)
    idx = torch.from_numpy(idx).cuda()
    import ctypes
    dims = B.make_dims(1024, cfg.D, cfg.E, cfg.k, cfg.I, True)
    ws = torch.empty(int(B.load().moe_backward_workspace_size(ctypes.byref(dims))), dtype=torch.uint8, device="cuda")
    eager = B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy, idx, True, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        captured = B.moe_backward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], dy, idx, True, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    for key, v in eager.items():
        if v is not None:
            assert torch.equal(v, captured[key]), key
    del g
