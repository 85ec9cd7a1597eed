"""moe_forward_noalloc: the forward pass for callers that cannot allocate device memory
(plugin hosts that pass only input and output buffers, runtimes that plan device memory up
front and forbid allocation once started).  Its scratch is a fixed 64 MiB array inside the
library.

Checked through the C ABI against moe_forward with a caller-owned workspace, on two calls
in a row (the second one runs on the scratch the first left behind), with the device error
word of those calls read back through moe_get_device_status_noalloc, plus the refusal of a
problem whose workspace does not fit.  Kept in a file that is collected last so a failure
here never hides the other tests; it passes alone in a fresh process as well.
"""
import pytest
import torch

from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import assert_y_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()


def test_noalloc_matches_forward_on_two_calls():
    cfg = inputs.CONFIGS["decode"]
    L = inputs.make_layer(cfg, T=256)
    G = {k: (v.cuda() if v is not None else None) for k, v in L.items()}
    for T in (256, 32):   # second call: smaller problem over the first call's leftovers
        x = G["x"][:T].contiguous()
        ref = B.moe_forward(x, G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, cfg.norm_topk_prob)
        got = B.moe_forward_noalloc(x, G["W_r"], G["W_gate_up"], G["W_down"], cfg.k,
                                    cfg.norm_topk_prob)
        torch.cuda.synchronize()
        assert_y_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), f"noalloc T={T}")
        assert torch.equal(got, ref)          # same kernels, same order: bitwise equal
        assert B.moe_get_device_status_noalloc() == B.MOE_OK


def test_noalloc_refuses_problems_larger_than_its_scratch():
    cfg = inputs.CONFIGS["decode"]
    T = 4096
    dims = B.make_dims(T, cfg.D, cfg.E, cfg.k, cfg.I)
    assert B.moe_workspace_size(dims) > 64 << 20
    x = torch.zeros(T, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_r = torch.zeros(cfg.E, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_gu = torch.zeros(cfg.E, 2 * cfg.I, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_dn = torch.zeros(cfg.E, cfg.D, cfg.I, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_forward_noalloc(x, W_r, W_gu, W_dn, cfg.k)
    assert ei.value.status == B.MOE_ERR_WORKSPACE
