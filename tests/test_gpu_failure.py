"""Failure detection on the GPU, made on the host (no fault, no trap, no unbounded wait).

* A bad routing input: moe_permute given an expert index outside [0, E).  The kernels skip
  that assignment and record it in the device error word; moe_get_device_status reports
  MOE_ERR_INVALID_ARG, and the next call on the same workspace starts clean.
* The watchdog: MOE_DIAG_UNSIGNALLED_HANDOFF points the down GEMM's per-expert hand-off
  wait at counters that no kernel increments (a flag that nothing sets) and wait_limit_us
  bounds every device wait at 20 ms.  The kernels give up, wind down (TMEM released, no copy
  in flight) and moe_get_device_status reports MOE_ERR_DEVICE_TIMEOUT; a normal call on the
  same workspace then runs correctly, so the context stayed usable.
* The decode kernel's watchdog: MOE_DIAG_DECODE_BARRIER makes its grid-wide barrier wait
  for one block more than the grid has; the same report and recovery.
"""
import time

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()


@pytest.mark.parametrize("T,k,E", [(40, 4, 16), (3000, 8, 128)])   # one block / multi-block
def test_permute_reports_out_of_range_expert(T, k, E):
    g = torch.Generator().manual_seed(T + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    bad = idx.clone()
    bad[T // 2, 1] = E                      # one index past the last expert
    dims = B.make_dims(T, 128, E, k, 128)
    ws = B.workspace(dims)
    out = B.moe_permute(bad.cuda(), E, 1, ws=ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_INVALID_ARG
    # the skipped assignment is missing from the counts; every other one is placed
    counts = out["counts"].cpu().numpy()
    expect = np.bincount(idx.numpy().reshape(-1), minlength=E)
    expect[idx[T // 2, 1]] -= 1
    assert np.array_equal(counts, expect)
    # the next call on the same workspace clears the word and is exact
    out = B.moe_permute(idx.cuda(), E, 1, ws=ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    c, off, rt, sr = O.permute(idx.numpy(), E, 1)
    assert np.array_equal(out["counts"].cpu().numpy(), c)
    assert np.array_equal(out["slot_row"].cpu().numpy(), sr)


def test_watchdog_reports_timeout_and_device_stays_usable():
    cfg = inputs.CONFIGS["decode"]
    L = inputs.make_layer(cfg, T=8)
    G = {k_: (v.cuda() if v is not None else None) for k_, v in L.items()}
    dims = B.make_dims(8, cfg.D, cfg.E, cfg.k, cfg.I)
    ws = B.workspace(dims)
    ref = B.moe_forward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    ref = ref.cpu()
    t0 = time.perf_counter()
    B.moe_forward_ex(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws,
                     wait_limit_us=20000, diag=B.MOE_DIAG_UNSIGNALLED_HANDOFF)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 < 1.9      # ended by the 20 ms limits, not the 2 s default
    y = B.moe_forward(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    assert torch.equal(y.cpu(), ref)


def test_decode_kernel_watchdog():
    """MOE_DIAG_DECODE_BARRIER: the decode kernel's grid barrier waits for a block that does
    not exist; every block gives up after the 20 ms limit, the call reports
    MOE_ERR_DEVICE_TIMEOUT, and the next call on the same workspace is exact again."""
    cfg = inputs.CONFIGS["decode"]
    L = inputs.make_layer(cfg, T=1)
    G = {k_: (v.cuda() if v is not None else None) for k_, v in L.items()}
    dims = B.make_dims(1, cfg.D, cfg.E, cfg.k, cfg.I)
    ws = B.workspace(dims)
    ref = B.moe_forward_ex(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws, path="decode")
    assert B.moe_get_device_status(ws) == B.MOE_OK
    ref = ref.cpu()
    t0 = time.perf_counter()
    B.moe_forward_ex(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws,
                     wait_limit_us=20000, diag=B.MOE_DIAG_DECODE_BARRIER)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 < 1.9
    y = B.moe_forward_ex(G["x"], G["W_r"], G["W_gate_up"], G["W_down"], cfg.k, ws=ws, path="decode")
    assert B.moe_get_device_status(ws) == B.MOE_OK
    assert torch.equal(y.cpu(), ref)
    # where the decode kernel does not apply the diagnostic is refused
    L8 = inputs.make_layer(cfg, T=8)
    with pytest.raises(B.MoeError) as ei:
        B.moe_forward_ex(L8["x"].cuda(), G["W_r"], G["W_gate_up"], G["W_down"], cfg.k,
                         diag=B.MOE_DIAG_DECODE_BARRIER)
    assert ei.value.status == B.MOE_ERR_UNSUPPORTED


def test_watchdog_diagnostic_needs_the_handoff():
    cfg = inputs.CONFIGS["prefill"]
    T = 2048                              # T*k > 32*E: the wide tiles have no hand-off wait
    x = torch.zeros(T, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_r = torch.zeros(cfg.E, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_gu = torch.zeros(cfg.E, 2 * cfg.I, cfg.D, dtype=torch.bfloat16, device="cuda")
    W_dn = torch.zeros(cfg.E, cfg.D, cfg.I, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_forward_ex(x, W_r, W_gu, W_dn, cfg.k, diag=B.MOE_DIAG_UNSIGNALLED_HANDOFF)
    assert ei.value.status == B.MOE_ERR_UNSUPPORTED
