"""moe_aux_loss (the Switch balance loss and its gradient with respect to the router logits)
on the GPU against the oracle's FP64 evaluation of the same definition.

Inputs are each configuration's own routing, made by the oracle's router and selection from
the seeded layer (FP32 logits and the top-k indices) and given to both sides: decode T=256,
prefill T=8192, zipf (E=512, k=10, Zipf router bias), tiny (E=8, tie rows).

Tolerances, from the FP32 arithmetic: P_e is a sum of T probabilities (each a few ulp off)
added in ~T/148 + 148 steps, f_e is exact up to one rounding, the loss sums E products: a
relative error below ~5e-5 in the worst case, so the loss is checked to 1e-4 relative.  Each
gradient entry p (f_e - q) carries those errors on q and p; it is checked to 1e-4 of the
largest gradient entry.
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


def routing(name, T=None):
    cfg, L, G = layer(name, T)
    logits, idx, _ = O.route(L["x"], L["W_r"], cfg.k, cfg.norm_topk_prob, bias=L.get("bias"))
    return cfg, torch.from_numpy(logits).cuda(), torch.from_numpy(idx).cuda()


@pytest.mark.parametrize("name,T", [("tiny", None), ("decode", 256), ("prefill", None), ("zipf", None)])
def test_aux_loss_against_oracle(name, T):
    cfg, logits, idx = routing(name, T)
    alpha = 0.001
    loss, d = B.moe_aux_loss(logits, idx, alpha)
    torch.cuda.synchronize()
    ref_loss, ref_d = O.aux_loss(logits.cpu().numpy(), idx.cpu().numpy(), alpha)
    got = float(loss.cpu()[0])
    assert abs(got - ref_loss) <= 1e-4 * abs(ref_loss), (got, ref_loss)
    d = d.cpu().numpy().astype(np.float64)
    scale = np.abs(ref_d).max()
    assert np.abs(d - ref_d).max() <= 1e-4 * scale, (np.abs(d - ref_d).max(), scale)
    assert np.abs(d.sum(axis=1)).max() <= 1e-5 * scale * logits.shape[1]   # rows sum to ~0
    print(f"{name}: loss {got:.6e} (oracle {ref_loss:.6e}), max |dL| {scale:.3e}")


def test_aux_loss_deterministic_and_loss_only():
    cfg, logits, idx = routing("prefill")
    l1, d1 = B.moe_aux_loss(logits, idx, 0.01)
    l2, d2 = B.moe_aux_loss(logits, idx, 0.01)
    l3, d3 = B.moe_aux_loss(logits, idx, 0.01, with_grad=False)
    torch.cuda.synchronize()
    assert torch.equal(l1, l2) and torch.equal(d1, d2) and torch.equal(l1, l3) and d3 is None


def test_aux_loss_balanced_and_uniform_cases():
    """The closed forms of the pins, on the GPU: equal logits give alpha*k for any routing,
    routing every expert equally often gives alpha*k for any logits."""
    T, E, k = 1024, 64, 4
    g = torch.Generator().manual_seed(2)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).cuda()
    flat = torch.full((T, E), 0.5, dtype=torch.float32, device="cuda")
    loss, _ = B.moe_aux_loss(flat, idx, 0.25)
    assert abs(float(loss.cpu()[0]) - 0.25 * k) <= 1e-6
    bal = torch.tensor([[(t * k + j) % E for j in range(k)] for t in range(T)], dtype=torch.int32).cuda()
    logits = torch.randn(T, E, generator=g).cuda()
    loss, _ = B.moe_aux_loss(logits, bal, 0.25)
    assert abs(float(loss.cpu()[0]) - 0.25 * k) <= 1e-5


def test_aux_loss_workspace_too_small():
    cfg, logits, idx = routing("tiny")
    n = B.load().moe_aux_loss_workspace_size(logits.shape[0], logits.shape[1])
    small = torch.empty(n - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_aux_loss(logits, idx, 0.1, ws=small)
    assert e.value.status == B.MOE_ERR_WORKSPACE
