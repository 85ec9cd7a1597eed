"""The C-ABI library on the host: it loads, exports every function the header declares,
sizes workspaces, names statuses, and rejects bad arguments before enqueuing anything.

Calls here that pass made-up device addresses only run when no GPU is present: they must be
rejected by validation (or, with valid arguments, fail at the first CUDA call) and never
reach a kernel.
"""
import ctypes
import subprocess

import pytest
import torch

from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200.build import LIB, build

no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="made-up device addresses: CPU-only test")


@pytest.fixture(scope="module")
def lib():
    build()
    return B.load()


def test_library_exports_every_declared_function(lib):
    declared = B.header_functions()
    assert set(declared) == {"moe_workspace_size", "moe_route", "moe_permute", "moe_forward",
                             "moe_forward_ex", "moe_forward_noalloc", "moe_get_device_status",
                             "moe_get_device_status_noalloc", "moe_status_string", "moe_last_cuda_error",
                             "moe_quantize_fp8_rows", "moe_forward_path", "moe_aux_loss",
                             "moe_aux_loss_workspace_size", "moe_backward", "moe_backward_workspace_size"}
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared:
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_is_sm100a_only_and_self_contained(lib):
    out = subprocess.run(["ldd", LIB], capture_output=True, text=True, check=True).stdout
    assert "libcudart" not in out and "libcuda.so" not in out   # static runtime, driver via entry point
    assert "libtorch" not in out and "python" not in out


def test_status_strings(lib):
    names = [B.status_string(s) for s in range(6)]
    assert names == ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_WORKSPACE",
                     "MOE_ERR_CUDA", "MOE_ERR_DEVICE_TIMEOUT"]
    assert B.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_size_valid_and_invalid(lib):
    d = B.make_dims(64, 256, 8, 2, 128)
    n = B.moe_workspace_size(d)
    assert n > 0 and n % 256 == 0
    assert B.moe_workspace_size(B.make_dims(128, 256, 8, 2, 128)) > n
    for bad in [B.make_dims(0, 256, 8, 2, 128), B.make_dims(64, 200, 8, 2, 128),
                B.make_dims(64, 256, 8, 2, 100), B.make_dims(64, 256, 513, 2, 128),
                B.make_dims(64, 256, 8, 9, 128), B.make_dims(64, 256, 32, 17, 128),
                B.make_dims(64, 256, 8, 2, 128, tile_m=0), B.make_dims(64, 256, 8, 2, 128, tile_m=300)]:
        assert B.moe_workspace_size(bad) == 0
    d = B.make_dims(64, 256, 8, 2, 128, norm_topk_prob=True)
    d.norm_topk_prob = 2
    assert B.moe_workspace_size(d) == 0
    # a shared expert adds rows and slots
    o = B.moe_opts()
    o.shared_gate_up, o.shared_down, o.I_s = 1 << 20, 2 << 20, 256
    assert B.moe_workspace_size(B.make_dims(64, 256, 8, 2, 128), o) > n
    o.I_s = 100
    assert B.moe_workspace_size(B.make_dims(64, 256, 8, 2, 128), o) == 0


FAKE = 1 << 24   # aligned made-up addresses; never dereferenced (validation fails first)


def _fwd(lib, dims, ws_bytes, x=FAKE, out=FAKE + (1 << 20), ws=FAKE + (2 << 20), opts=None):
    p = lambda v: ctypes.c_void_p(v) if v else None
    return lib.moe_forward_ex(p(x), p(FAKE), p(FAKE), p(FAKE), ctypes.byref(dims),
                              ctypes.byref(opts) if opts else None, p(out), p(ws), ws_bytes, None)


@no_gpu
def test_forward_rejects_bad_arguments_before_launch(lib):
    d = B.make_dims(64, 256, 8, 2, 128)
    n = B.moe_workspace_size(d)
    assert _fwd(lib, d, n, x=0) == B.MOE_ERR_INVALID_ARG
    assert _fwd(lib, d, n, ws=0) == B.MOE_ERR_INVALID_ARG
    assert _fwd(lib, d, n, x=FAKE + 2) == B.MOE_ERR_INVALID_ARG          # misaligned
    assert _fwd(lib, d, n, ws=FAKE + 16) == B.MOE_ERR_INVALID_ARG        # workspace not 256-aligned
    assert _fwd(lib, d, n, out=FAKE) == B.MOE_ERR_INVALID_ARG            # out aliases x
    assert _fwd(lib, d, n - 256) == B.MOE_ERR_WORKSPACE
    assert _fwd(lib, B.make_dims(64, 256, 8, 9, 128), n) == B.MOE_ERR_UNSUPPORTED
    assert _fwd(lib, B.make_dims(0, 256, 8, 2, 128), n) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.path = 7
    assert _fwd(lib, d, n, opts=o) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.shared_gate_up = FAKE                     # shared expert without its down projection
    o.I_s = 128
    assert _fwd(lib, d, n, opts=o) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.n_stage_events = 3
    assert _fwd(lib, d, n, opts=o) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.diag = 3                                  # no such diagnostic
    assert _fwd(lib, d, n, opts=o) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.slot_row_out = FAKE + 2                   # misaligned routing-table output
    assert _fwd(lib, d, n, opts=o) == B.MOE_ERR_INVALID_ARG
    o = B.moe_opts()
    o.diag = B.MOE_DIAG_UNSIGNALLED_HANDOFF     # wide shape (T*k > 32*E): no hand-off wait
    wide = B.make_dims(512, 256, 8, 2, 128)
    assert _fwd(lib, wide, B.moe_workspace_size(wide), opts=o) == B.MOE_ERR_UNSUPPORTED


@no_gpu
def test_forward_path_query_without_a_device(lib):
    """moe_forward_path validates like moe_forward_ex; the choice itself needs the device's SM
    count, so without a GPU a valid query reports a CUDA failure."""
    d = B.make_dims(2, 256, 8, 2, 128)
    out = ctypes.c_int(-1)
    assert lib.moe_forward_path(ctypes.byref(d), None, ctypes.byref(out)) == B.MOE_ERR_CUDA
    o = B.moe_opts()
    o.path = 7
    assert lib.moe_forward_path(ctypes.byref(d), ctypes.byref(o), ctypes.byref(out)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_path(ctypes.byref(B.make_dims(2, 256, 8, 9, 128)), None,
                                ctypes.byref(out)) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_forward_path(ctypes.byref(d), None, None) == B.MOE_ERR_INVALID_ARG


@no_gpu
def test_no_cpu_fallback(lib):
    """With valid arguments and no GPU the library reports a CUDA failure (and keeps the
    CUDA error code for diagnostics); it never computes anything on the host."""
    d = B.make_dims(64, 256, 8, 2, 128)
    assert _fwd(lib, d, B.moe_workspace_size(d)) == B.MOE_ERR_CUDA
    assert B.moe_last_cuda_error() != 0
    p = ctypes.c_void_p
    assert lib.moe_route(p(FAKE), p(FAKE), None, ctypes.byref(d), None, p(FAKE), p(FAKE),
                         p(FAKE), B.moe_workspace_size(d), None) == B.MOE_ERR_CUDA


@no_gpu
def test_permute_and_route_validation(lib):
    d = B.make_dims(64, 256, 8, 2, 128, tile_m=4)
    n = B.moe_workspace_size(d)
    p = ctypes.c_void_p
    cap = 64 * 2 + 8 * 3
    args = lambda cap_, ws_: (p(FAKE), None, None, ctypes.byref(d), p(FAKE), p(FAKE), p(FAKE),
                              p(FAKE), None, None, cap_, p(FAKE), ws_, None)
    assert lib.moe_permute(*args(cap - 1, n)) == B.MOE_ERR_INVALID_ARG   # cap too small
    assert lib.moe_permute(*args(cap, n - 256)) == B.MOE_ERR_WORKSPACE
    assert lib.moe_route(None, p(FAKE), None, ctypes.byref(d), None, p(FAKE), p(FAKE), p(FAKE), n,
                         None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_get_device_status(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_get_device_status_noalloc(None) == B.MOE_ERR_CUDA     # no device here


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        B.load()


@no_gpu
def test_aux_loss_validation_without_a_device(lib):
    """moe_aux_loss validates before enqueuing; with valid arguments and no GPU it reports a
    CUDA failure (no host fallback)."""
    p = ctypes.c_void_p
    n = lib.moe_aux_loss_workspace_size(64, 8)
    assert n > 0 and lib.moe_aux_loss_workspace_size(64, 513) == 0
    args = lambda T=64, E=8, k=2, ws=FAKE, nb=n, lg=FAKE: (p(lg), p(FAKE), T, E, k, ctypes.c_float(0.01), p(FAKE),
                                                          None, p(ws), nb, None)
    assert lib.moe_aux_loss(*args(T=0)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_loss(*args(k=9)) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_aux_loss(*args(E=513)) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_aux_loss(*args(lg=0)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_loss(*args(ws=FAKE + 16)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_loss(*args(nb=n - 4)) == B.MOE_ERR_WORKSPACE
    assert lib.moe_aux_loss(*args()) == B.MOE_ERR_CUDA


@no_gpu
def test_backward_validation_without_a_device(lib):
    """moe_backward validates before enqueuing (shape, pointers, alignment, workspace); with
    valid arguments and no GPU it reports a CUDA failure (no host fallback)."""
    p = ctypes.c_void_p
    dims = B.make_dims(64, 256, 8, 2, 128, True)
    n = lib.moe_backward_workspace_size(ctypes.byref(dims))
    assert n > lib.moe_workspace_size(ctypes.byref(dims), None) > 0
    assert lib.moe_backward_workspace_size(ctypes.byref(B.make_dims(64, 200, 8, 2, 128, True))) == 0

    def call(d=dims, x=FAKE, dx=FAKE, ws=FAKE, nb=n, residual=0, idx=FAKE):
        return lib.moe_backward(p(x), p(FAKE), None, p(FAKE), p(FAKE), p(FAKE), p(idx), None, residual,
                                ctypes.byref(d), p(dx), p(FAKE), None, p(FAKE), p(FAKE), None, None, p(ws), nb, None)
    assert call(d=B.make_dims(0, 256, 8, 2, 128, True)) == B.MOE_ERR_INVALID_ARG
    assert call(d=B.make_dims(64, 200, 8, 2, 128, True)) == B.MOE_ERR_UNSUPPORTED
    assert call(x=0) == B.MOE_ERR_INVALID_ARG
    assert call(idx=0) == B.MOE_ERR_INVALID_ARG
    assert call(dx=FAKE + 4) == B.MOE_ERR_INVALID_ARG
    assert call(ws=FAKE + 16) == B.MOE_ERR_INVALID_ARG
    assert call(residual=2) == B.MOE_ERR_INVALID_ARG
    assert call(nb=n - 256) == B.MOE_ERR_WORKSPACE
    assert call() == B.MOE_ERR_CUDA
