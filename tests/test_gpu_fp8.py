"""FP8 weight-only experts on the GPU against the oracle.

* moe_quantize_fp8_rows: every byte and every scale bit-exact against the oracle's
  quantiser (the same reading: FP32 row scale amax / 448, FP32 quotient, E4M3 nearest-even
  with saturation), on the decode shape's full expert tensors plus edge rows.
* moe_forward_ex with FP8 experts: routing as in the bf16 tests (the router stays bf16);
  the output against the oracle evaluating the definition with the dequantised weights
  (weight = scale[row] * value(q)), with the block's output criterion.
* One token runs on the one-token kernel with FP8 weights: against the oracle (the sweep's
  T=1) and against the grouped FP8 path on the same token.
* The cases the FP8 path refuses (a shared expert, wider batches) return MOE_ERR_UNSUPPORTED.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import W_ATOL, assert_block_output, assert_y_close, check_routing, logit_deltas

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, O.cpu_threads_available()))


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()
    O.build()


_q = {}


def decode_fp8():
    """The decode layer with its experts quantised by the library (checked against the oracle
    in test_quantize_bit_exact)."""
    if "decode" not in _q:
        cfg = inputs.CONFIGS["decode"]
        L = inputs.make_layer(cfg, T=256)
        G = {k: (v.cuda() if v is not None else None) for k, v in L.items()}
        q_gu, s_gu = B.moe_quantize_fp8_rows(G["W_gate_up"])
        q_dn, s_dn = B.moe_quantize_fp8_rows(G["W_down"])
        torch.cuda.synchronize()
        _q["decode"] = (cfg, L, G, dict(W_gate_up_fp8=q_gu, gate_up_scale=s_gu, W_down_fp8=q_dn,
                                        down_scale=s_dn))
    return _q["decode"]


def test_quantize_bit_exact():
    cfg, L, G, F = decode_fp8()
    for name, qn, sn in (("W_gate_up", "W_gate_up_fp8", "gate_up_scale"), ("W_down", "W_down_fp8", "down_scale")):
        q_o, s_o = O.quantize_fp8_rows(L[name])
        assert np.array_equal(F[sn].cpu().numpy().view(np.uint32), s_o.view(np.uint32)), name
        assert np.array_equal(F[qn].cpu().numpy(), q_o), name
    # edge rows: zeros, one large value, tiny values (E4M3 subnormals), exact ties, signed zeros
    g = torch.Generator().manual_seed(11)
    W = (torch.randn(40, 512, generator=g) * 0.02)
    W[0] = 0
    W[1, 7] = 3.0e4
    W[2] = W[2] * 1e-6
    W[2, 0] = 1.0
    W[3] = torch.tensor([448.0, 0.5 * 2 ** -9, 1.5 * 2 ** -9, 1.0625, 1.1875, -0.0] * 85 + [1.0, 2.0])[:512]
    W[4] = -W[4]
    Wb = W.to(torch.bfloat16)
    q, s = B.moe_quantize_fp8_rows(Wb.cuda())
    q_o, s_o = O.quantize_fp8_rows(Wb)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_o)


def run_fp8(cfg, G, F, x, residual=None):
    T, E, k = x.shape[0], G["W_r"].shape[0], cfg.k
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    y32 = torch.empty(x.shape, dtype=torch.float32, device="cuda")
    out = B.moe_forward_ex(x, G["W_r"], None, None, k, cfg.norm_topk_prob, residual=residual,
                           logits_out=logits, topk_idx_out=idx, topk_w_out=w, out_f32=y32, **F)
    torch.cuda.synchronize()
    return out.cpu(), y32.cpu(), idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()


@pytest.mark.parametrize("T", [1, 8, 32, 128, 256])
def test_forward_fp8_decode_sweep(T):
    cfg, L, G, F = decode_fp8()
    x_cpu = L["x"][:T].contiguous()
    y, y32, idx, w, logits = run_fp8(cfg, G, F, x_cpu.cuda())
    rows = np.arange(T, dtype=np.int32)
    o_idx, o_w = O.select(logits, cfg.k, cfg.norm_topk_prob)
    assert np.array_equal(o_idx, idx)
    assert np.abs(o_w - w).max() <= W_ATOL
    ol = O.router_logits(x_cpu, L["W_r"])
    oi, _ = O.select(ol, cfg.k, cfg.norm_topk_prob)
    delta = logit_deltas(x_cpu, L["W_r"], ol)
    assert (np.abs(logits - ol) <= delta + 1e-30).all()
    check_routing(idx, oi, ol, delta, cfg.k)
    # the output for the GPU's (checked) routing, with the dequantised experts
    y_ref = O.combine_rows_fp8(x_cpu, idx, w, rows, F["W_gate_up_fp8"], F["gate_up_scale"],
                               F["W_down_fp8"], F["down_scale"], threads=THREADS)
    assert_block_output(y, y32, y_ref, f"fp8 decode T={T}")


def test_forward_fp8_residual_and_status():
    cfg, L, G, F = decode_fp8()
    T = 8
    x_cpu = L["x"][:T].contiguous()
    res_cpu = inputs.normal_bf16((T, cfg.D), 1.0, 77)
    ws = B.workspace(B.make_dims(T, cfg.D, cfg.E, cfg.k, cfg.I), B.make_opts(**F))
    y32 = torch.empty(T, cfg.D, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, cfg.k, dtype=torch.float32, device="cuda")
    out = B.moe_forward_ex(x_cpu.cuda(), G["W_r"], None, None, cfg.k, True, ws=ws, residual=res_cpu.cuda(),
                           out_f32=y32, topk_idx_out=idx, topk_w_out=w, **F)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    y_ref = O.combine_rows_fp8(x_cpu, idx.cpu().numpy(), w.cpu().numpy(), np.arange(T, dtype=np.int32),
                               F["W_gate_up_fp8"], F["gate_up_scale"], F["W_down_fp8"], F["down_scale"],
                               residual=res_cpu, threads=THREADS)
    assert_block_output(out.cpu(), y32.cpu(), y_ref, "fp8 residual")


def test_fp8_refused_where_unsupported():
    cfg, L, G, F = decode_fp8()
    # a batch past the narrow-tile regime (T*k > 32*E)
    x = torch.zeros(600, cfg.D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(x, G["W_r"], None, None, cfg.k, True, **F)
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    # with a shared expert
    sgu = torch.zeros(2 * 128, cfg.D, dtype=torch.bfloat16, device="cuda")
    sdn = torch.zeros(cfg.D, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(G["x"][:4].contiguous(), G["W_r"], None, None, cfg.k, True,
                         shared_gate_up=sgu, shared_down=sdn, **F)
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    # half of the FP8 arguments (with a workspace, so that the forward itself validates)
    ws = B.workspace(B.make_dims(4, cfg.D, cfg.E, cfg.k, cfg.I))
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(G["x"][:4].contiguous(), G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, True,
                         ws=ws, W_gate_up_fp8=F["W_gate_up_fp8"])
    assert e.value.status == B.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("t", [0, 5])
def test_fp8_one_token_kernel_matches_grouped(t):
    """One token goes through the one-token kernel (AUTO's choice); the grouped FP8 path on the
    same token gives the same routing bit for bit and the output within the tolerance."""
    cfg, L, G, F = decode_fp8()
    x = G["x"][t:t + 1].contiguous()
    assert B.moe_forward_path(B.make_dims(1, cfg.D, cfg.E, cfg.k, cfg.I), B.make_opts(**F)) == "decode"
    outs = {}
    for path in ("decode", "grouped"):
        idx = torch.empty(1, cfg.k, dtype=torch.int32, device="cuda")
        w = torch.empty(1, cfg.k, dtype=torch.float32, device="cuda")
        y = B.moe_forward_ex(x, G["W_r"], None, None, cfg.k, cfg.norm_topk_prob, topk_idx_out=idx,
                             topk_w_out=w, path=path, **F)
        torch.cuda.synchronize()
        outs[path] = (y.cpu(), idx.cpu().numpy(), w.cpu().numpy())
    assert (outs["decode"][1] == outs["grouped"][1]).all() and (outs["decode"][2] == outs["grouped"][2]).all()
    assert_y_close(outs["decode"][0].double().numpy(), outs["grouped"][0].double().numpy(), f"fp8 token {t}")
