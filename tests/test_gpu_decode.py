"""The decode kernel (MOE_PATH_DECODE: the whole block in one kernel for one token) on the GPU.

* Against the oracle (routing bit-exact on the GPU's logits, logits within the FP32 bound,
  outputs under the block's criterion): several tokens of the decode workload one at a time,
  the keras and zipf router shapes (E = 60 / 512 with a Zipf bias), k = 1, k = E, E = 1,
  k = 16 of 512, norm off, a router bias that sends the token to one expert, every tie row of
  the tiny config, a residual (also updated in place), D = 128 (more SMs than output rows),
  a zero token.
* Against the grouped path on the same token: the same logits, experts and weights bit for
  bit (the two routers sum in the same order), outputs within the output tolerance.
* Bitwise reruns; what AUTO picks; what the path refuses.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import assert_y_close
from tests.test_gpu_parity import _small_layer, compare_block, layer, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()
    O.build()


def f64(y):
    return y.double().numpy()


def test_auto_picks_decode_for_one_token():
    cfg = inputs.CONFIGS["decode"]
    assert B.moe_forward_path(B.make_dims(1, cfg.D, cfg.E, cfg.k, cfg.I)) == "decode"
    assert B.moe_forward_path(B.make_dims(2, cfg.D, cfg.E, cfg.k, cfg.I)) == "grouped"
    dims = B.make_dims(1, cfg.D, cfg.E, cfg.k, cfg.I)
    assert B.moe_forward_path(dims, B.make_opts(path="grouped")) == "grouped"
    counts = torch.empty(cfg.E, dtype=torch.int32, device="cuda")
    assert B.moe_forward_path(dims, B.make_opts(expert_counts_out=counts)) == "grouped"
    assert B.moe_forward_path(B.make_dims(1, 4096, cfg.E, cfg.k, cfg.I)) == "grouped"   # D > 2048


@pytest.mark.parametrize("t", [0, 1, 77, 255])
def test_decode_workload_tokens(t):
    cfg, L, G = layer("decode", 256)
    x = L["x"][t:t + 1].contiguous()
    compare_block(cfg, L, G, [0], path="decode", x_cpu=x, what=f"decode kernel token {t}")


@pytest.mark.parametrize("name", ["keras", "zipf_router"])
def test_decode_other_shapes(name):
    if name == "zipf_router":   # E = 512, k = 10, Zipf router bias; no shared expert
        cfg = inputs.CONFIGS["zipf"]
        bias = inputs.zipf_bias(cfg.E, cfg.zipf_s, cfg.seed)
        c, L, G = _small_layer(1, D=cfg.D, E=cfg.E, k=cfg.k, I=cfg.I, seed=cfg.seed, bias=bias)
        compare_block(c, L, G, [0], path="decode", what="E=512 k=10 bias")
        return
    cfg, L, G = layer(name, None)
    for t in (0, 4095):
        x = L["x"][t:t + 1].contiguous()
        compare_block(cfg, L, G, [0], path="decode", x_cpu=x, what=f"{name} token {t}")


@pytest.mark.parametrize("E,k,norm", [(16, 1, True), (8, 8, True), (16, 4, False), (1, 1, True), (512, 16, True)])
def test_decode_k_E_norm(E, k, norm):
    cfg, L, G = _small_layer(1, E=E, k=k)
    compare_block(cfg, L, G, [0], path="decode", k=k, norm=norm, what=f"E={E} k={k} norm={norm}")


def test_decode_all_on_one_expert():
    bias = torch.zeros(16)
    bias[3] = 100.0
    cfg, L, G = _small_layer(1, bias=bias)
    r = compare_block(cfg, L, G, [0], path="decode", what="one expert")
    assert r["idx"][0, 0] == 3


@pytest.mark.parametrize("row", sorted(inputs.TINY_TIES))
def test_decode_tie_rows(row):
    cfg, L, G = layer("tiny")
    x = L["x"][row:row + 1].contiguous()
    r = compare_block(cfg, L, G, [0], path="decode", x_cpu=x, what=f"tie row {row}")
    assert tuple(r["idx"][0].tolist()) == inputs.TINY_TIES[row][2]
    if row == 63:
        assert (r["y"][0] == 0).all()


def test_decode_residual_in_place_and_small_D():
    cfg, L, G = _small_layer(1, D=128, E=8, k=2, I=128)   # 128 output rows on ~148 blocks
    res = torch.randn(1, 128, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    compare_block(cfg, L, G, [0], path="decode", residual_cpu=res, what="residual D=128")
    # out aliasing the residual: the block updates the residual stream in place
    y_sep, _, _, _ = run_forward(cfg, G, path="decode", residual=res.cuda())
    buf = res.cuda().clone()
    B.moe_forward_ex(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, True, out=buf, residual=buf,
                     path="decode")
    torch.cuda.synchronize()
    assert torch.equal(buf.cpu(), y_sep)


def test_decode_zero_input():
    cfg, L, G = _small_layer(1)
    res = torch.randn(1, 256, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    y, idx, w, _ = run_forward(cfg, G, path="decode", x=torch.zeros(1, 256, dtype=torch.bfloat16, device="cuda"),
                               residual=res.cuda())
    assert torch.equal(y, res)                                 # block(0) = 0 exactly
    assert (idx == np.arange(cfg.k)[None, :]).all()


@pytest.mark.parametrize("t", [0, 3])
def test_decode_matches_grouped(t):
    cfg, L, G = layer("decode", 8)
    x = G["x"][t:t + 1].contiguous()
    yd, id_, wd, ld = run_forward(cfg, G, path="decode", x=x)
    yg, ig, wg, lg = run_forward(cfg, G, path="grouped", x=x)
    assert (ld == lg).all() and (id_ == ig).all() and (wd == wg).all()
    assert_y_close(f64(yd), f64(yg), f"decode vs grouped token {t}")


def test_decode_deterministic():
    cfg, L, G = layer("decode", 8)
    x = G["x"][5:6].contiguous()
    runs = [run_forward(cfg, G, path="decode", x=x) for _ in range(3)]
    for y, i, w, l in runs[1:]:
        assert torch.equal(y, runs[0][0]) and (i == runs[0][1]).all() and (w == runs[0][2]).all()


def test_decode_refusals():
    cfg, L, G = layer("decode", 8)
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(G["x"][:2].contiguous(), G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, path="decode")
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    c2, L2, G2 = _small_layer(1, I_s=128)
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(G2["x"], G2["W_r"], G2["W_gate_up"], G2["W_down"], c2.k, path="decode",
                         shared_gate_up=G2["shared_gate_up"], shared_down=G2["shared_down"])
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    slot_row = torch.empty(1, c2.k, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_forward_ex(G2["x"], G2["W_r"], G2["W_gate_up"], G2["W_down"], c2.k, path="decode",
                         slot_row_out=slot_row)
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
