"""ctypes binding of ``libmoe_b200.so`` with the C ABI's own names.

Argument marshalling only: shapes are read from the tensors, pointers and the current CUDA
stream are handed to the library, and a non-zero status raises ``MoeError``.  Every step of
the computation runs in the library's kernels.  PyTorch supplies device memory (outputs and
the workspace) and streams.  If the library is missing this module raises instead of
falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe_b200.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT = range(6)
MOE_PATH_AUTO, MOE_PATH_GROUPED, MOE_PATH_DECODE = range(3)
PATHS = {"auto": MOE_PATH_AUTO, "grouped": MOE_PATH_GROUPED, "decode": MOE_PATH_DECODE}
MOE_DIAG_UNSIGNALLED_HANDOFF = 1
MOE_DIAG_DECODE_BARRIER = 2

_c_int, _vp, _sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t


class moe_dims(ctypes.Structure):
    _fields_ = [("T", _c_int), ("D", _c_int), ("E", _c_int), ("k", _c_int), ("I", _c_int),
                ("norm_topk_prob", _c_int), ("tile_m", _c_int)]


class moe_opts(ctypes.Structure):
    _fields_ = [("router_bias", _vp), ("shared_gate_up", _vp), ("shared_down", _vp),
                ("shared_gate", _vp), ("I_s", _c_int), ("residual", _vp), ("logits_out", _vp),
                ("topk_idx_out", _vp), ("topk_w_out", _vp), ("path", _c_int),
                ("stage_events", _vp), ("n_stage_events", _c_int), ("out_f32", _vp),
                ("expert_counts_out", _vp), ("slot_row_out", _vp), ("wait_limit_us", ctypes.c_uint),
                ("diag", _c_int), ("W_gate_up_fp8", _vp), ("gate_up_scale", _vp),
                ("W_down_fp8", _vp), ("down_scale", _vp)]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def load():
    """Load the library (once).  Raises when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_fp32_softmax_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        dp = ctypes.POINTER(moe_dims)
        op = ctypes.POINTER(moe_opts)
        lib.moe_workspace_size.argtypes = [dp, op]
        lib.moe_workspace_size.restype = _sz
        lib.moe_route.argtypes = [_vp, _vp, _vp, dp, _vp, _vp, _vp, _vp, _sz, _vp]
        lib.moe_permute.argtypes = [_vp, _vp, _vp, dp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _sz, _vp]
        lib.moe_forward.argtypes = [_vp, _vp, _vp, _vp, dp, _vp, _vp, _sz, _vp]
        lib.moe_forward_ex.argtypes = [_vp, _vp, _vp, _vp, dp, op, _vp, _vp, _sz, _vp]
        lib.moe_forward_noalloc.argtypes = [_vp, _vp, _vp, _vp, dp, _vp, _vp]
        lib.moe_get_device_status.argtypes = [_vp, _vp]
        lib.moe_get_device_status_noalloc.argtypes = [_vp]
        lib.moe_status_string.argtypes = [_c_int]
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_last_cuda_error.argtypes = []
        lib.moe_last_cuda_error.restype = _c_int
        lib.moe_quantize_fp8_rows.argtypes = [_vp, ctypes.c_int64, _c_int, _vp, _vp, _vp]
        lib.moe_forward_path.argtypes = [dp, op, ctypes.POINTER(_c_int)]
        lib.moe_aux_loss_workspace_size.argtypes = [_c_int, _c_int]
        lib.moe_aux_loss_workspace_size.restype = _sz
        lib.moe_aux_loss.argtypes = [_vp, _vp, _c_int, _c_int, _c_int, ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
        lib.moe_backward_workspace_size.argtypes = [dp]
        lib.moe_backward_workspace_size.restype = _sz
        lib.moe_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, dp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _sz, _vp]
        for n in ("moe_route", "moe_permute", "moe_forward", "moe_forward_ex", "moe_forward_noalloc",
                  "moe_get_device_status", "moe_get_device_status_noalloc", "moe_quantize_fp8_rows",
                  "moe_forward_path", "moe_aux_loss", "moe_backward"):
            getattr(lib, n).restype = _c_int
        _lib = lib
    return _lib


def header_functions():
    """Names of the functions ``include/moe_b200.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(moe_[a-z0-9_]+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


moe_status_string = status_string


def moe_last_cuda_error() -> int:
    return int(load().moe_last_cuda_error())


def _check(status, what):
    if status != MOE_OK:
        if status == MOE_ERR_CUDA:
            what = f"{what} (cudaError {moe_last_cuda_error()})"
        raise MoeError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, dims=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions")


def make_dims(T, D, E, k, I, norm_topk_prob=True, tile_m=1) -> moe_dims:
    return moe_dims(int(T), int(D), int(E), int(k), int(I), int(bool(norm_topk_prob)), int(tile_m))


def make_opts(router_bias=None, shared_gate_up=None, shared_down=None, shared_gate=None,
              residual=None, logits_out=None, topk_idx_out=None, topk_w_out=None, path="auto",
              stage_events=None, out_f32=None, expert_counts_out=None, slot_row_out=None,
              wait_limit_us=0, diag=0, W_gate_up_fp8=None, gate_up_scale=None, W_down_fp8=None,
              down_scale=None):
    o = moe_opts()
    o.router_bias = _ptr(router_bias)
    o.shared_gate_up = _ptr(shared_gate_up)
    o.shared_down = _ptr(shared_down)
    o.shared_gate = _ptr(shared_gate)
    o.I_s = int(shared_gate_up.shape[0] // 2) if shared_gate_up is not None else 0
    o.residual = _ptr(residual)
    o.logits_out = _ptr(logits_out)
    o.topk_idx_out = _ptr(topk_idx_out)
    o.topk_w_out = _ptr(topk_w_out)
    o.path = PATHS[path] if isinstance(path, str) else int(path)
    o.out_f32 = _ptr(out_f32)
    o.expert_counts_out = _ptr(expert_counts_out)
    o.slot_row_out = _ptr(slot_row_out)
    o.wait_limit_us = int(wait_limit_us)
    o.diag = int(diag)
    o.W_gate_up_fp8 = _ptr(W_gate_up_fp8)
    o.gate_up_scale = _ptr(gate_up_scale)
    o.W_down_fp8 = _ptr(W_down_fp8)
    o.down_scale = _ptr(down_scale)
    o._fp8 = (W_gate_up_fp8, W_down_fp8)   # shapes for the dims, and kept alive with the options
    o._events_keepalive = None
    if stage_events is not None:
        handles = (ctypes.c_void_p * len(stage_events))(*[ev.cuda_event for ev in stage_events])
        o._events_keepalive = handles
        o.stage_events = ctypes.cast(handles, ctypes.c_void_p)
        o.n_stage_events = len(stage_events)
    return o


def moe_workspace_size(dims: moe_dims, opts: moe_opts | None = None) -> int:
    return int(load().moe_workspace_size(ctypes.byref(dims), ctypes.byref(opts) if opts else None))


def moe_forward_path(dims: moe_dims, opts: moe_opts | None = None) -> str:
    """The path moe_forward_ex takes for these arguments: "decode" or "grouped"."""
    out = _c_int(-1)
    _check(load().moe_forward_path(ctypes.byref(dims), ctypes.byref(opts) if opts else None, ctypes.byref(out)),
           "moe_forward_path")
    return {MOE_PATH_DECODE: "decode", MOE_PATH_GROUPED: "grouped"}[out.value]


def moe_aux_loss(logits, topk_idx, alpha=1.0, with_grad=True, ws=None, stream=None):
    """Switch balance loss (and its gradient with respect to the logits) -> (loss [1] f32,
    dlogits [T, E] f32 or None)."""
    _need(logits, "logits", torch.float32, 2)
    _need(topk_idx, "topk_idx", torch.int32, 2)
    T, E = logits.shape
    k = topk_idx.shape[1]
    lib = load()
    n = int(lib.moe_aux_loss_workspace_size(T, E))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_aux_loss_workspace_size")
    if ws is None:
        ws = torch.empty(n, dtype=torch.uint8, device=logits.device)
    loss = torch.empty(1, dtype=torch.float32, device=logits.device)
    d = torch.empty(T, E, dtype=torch.float32, device=logits.device) if with_grad else None
    _check(lib.moe_aux_loss(_ptr(logits), _ptr(topk_idx), T, E, k, float(alpha), _ptr(loss), _ptr(d), _ptr(ws),
                            ws.numel(), _stream(stream)), "moe_aux_loss")
    return loss, d


def moe_backward(x, W_r, W_gate_up, W_down, dy, topk_idx, norm_topk_prob=True, bias=None, dlogits_add=None,
                 residual=False, with_dbias=None, ws=None, stream=None):
    """Gradients of sum(dy * y) for the routing topk_idx -> dict of FP32 tensors dx [T, D],
    dW_r [E, D], dbias [E] (when a bias is given or with_dbias), dW_gate_up [E, 2I, D],
    dW_down [E, D, I], dlogits [T, E], dw [T, k]."""
    dims = _dims_of(x, W_r, W_gate_up, W_down, topk_idx.shape[1], norm_topk_prob)
    _need(dy, "dy", torch.bfloat16, 2)
    _need(topk_idx, "topk_idx", torch.int32, 2)
    T, D, E, k, I = dims.T, dims.D, dims.E, dims.k, dims.I
    lib = load()
    n = int(lib.moe_backward_workspace_size(ctypes.byref(dims)))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_backward_workspace_size")
    dev = x.device
    if ws is None:
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    f32 = lambda *s: torch.empty(*s, dtype=torch.float32, device=dev)
    out = dict(dx=f32(T, D), dW_r=f32(E, D), dW_gate_up=f32(E, 2 * I, D), dW_down=f32(E, D, I), dlogits=f32(T, E),
               dw=f32(T, k))
    out["dbias"] = f32(E) if (bias is not None or with_dbias) else None
    _check(lib.moe_backward(_ptr(x), _ptr(W_r), _ptr(bias), _ptr(W_gate_up), _ptr(W_down), _ptr(dy), _ptr(topk_idx),
                            _ptr(dlogits_add), int(bool(residual)), ctypes.byref(dims), _ptr(out["dx"]),
                            _ptr(out["dW_r"]), _ptr(out["dbias"]), _ptr(out["dW_gate_up"]), _ptr(out["dW_down"]),
                            _ptr(out["dlogits"]), _ptr(out["dw"]), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_backward")
    return out


def workspace(dims: moe_dims, opts: moe_opts | None = None, device=None) -> torch.Tensor:
    n = moe_workspace_size(dims, opts)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def moe_route(x, W_r, k, norm_topk_prob=True, bias=None, logits=None, ws=None, stream=None):
    """-> (logits [T, E] f32, topk_idx [T, k] int32, topk_w [T, k] f32)."""
    _need(x, "x", torch.bfloat16, 2)
    _need(W_r, "W_r", torch.bfloat16, 2)
    T, D = x.shape
    E = W_r.shape[0]
    dims = make_dims(T, D, E, k, 128, norm_topk_prob)
    if logits is None:
        logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(dims, device=x.device)
    _check(load().moe_route(_ptr(x), _ptr(W_r), _ptr(bias), ctypes.byref(dims), _ptr(logits),
                            _ptr(idx), _ptr(w), _ptr(ws), ws.numel(), _stream(stream)), "moe_route")
    return logits, idx, w


def moe_permute(topk_idx, E, tile_m=1, topk_w=None, x=None, want_x_perm=False, ws=None, stream=None):
    """-> dict(counts, offsets, row_token, slot_row, row_weight, x_perm)."""
    _need(topk_idx, "topk_idx", torch.int32, 2)
    T, k = topk_idx.shape
    D = x.shape[1] if x is not None else 128
    dims = make_dims(T, D, E, k, 128, True, tile_m)
    cap = T * k + E * (tile_m - 1)
    dev = topk_idx.device
    out = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               row_token=torch.empty(cap, dtype=torch.int32, device=dev),
               slot_row=torch.empty(T * k, dtype=torch.int32, device=dev),
               row_weight=torch.empty(cap, dtype=torch.float32, device=dev) if topk_w is not None else None,
               x_perm=torch.empty(cap, D, dtype=torch.bfloat16, device=dev) if want_x_perm else None)
    if ws is None:
        ws = workspace(dims, device=dev)
    _check(load().moe_permute(_ptr(topk_idx), _ptr(topk_w), _ptr(x), ctypes.byref(dims),
                              _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["row_token"]),
                              _ptr(out["slot_row"]), _ptr(out["row_weight"]), _ptr(out["x_perm"]),
                              cap, _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return out


def _dims_of(x, W_r, W_gate_up, W_down, k, norm_topk_prob, W_gate_up_fp8=None, W_down_fp8=None):
    _need(x, "x", torch.bfloat16, 2)
    _need(W_r, "W_r", torch.bfloat16, 2)
    if W_gate_up is None and W_gate_up_fp8 is not None:   # FP8 experts: shapes from the bytes
        _need(W_gate_up_fp8, "W_gate_up_fp8", torch.uint8, 3)
        _need(W_down_fp8, "W_down_fp8", torch.uint8, 3)
        W_gate_up = W_gate_up_fp8
    else:
        _need(W_gate_up, "W_gate_up", torch.bfloat16, 3)
        _need(W_down, "W_down", torch.bfloat16, 3)
    T, D = x.shape
    E, I2, _ = W_gate_up.shape
    return make_dims(T, D, E, k, I2 // 2, norm_topk_prob)


def moe_forward(x, W_r, W_gate_up, W_down, k, norm_topk_prob=True, out=None, ws=None, stream=None):
    dims = _dims_of(x, W_r, W_gate_up, W_down, k, norm_topk_prob)
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = workspace(dims, device=x.device)
    _check(load().moe_forward(_ptr(x), _ptr(W_r), _ptr(W_gate_up), _ptr(W_down), ctypes.byref(dims),
                              _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward")
    return out


def moe_forward_ex(x, W_r, W_gate_up, W_down, k, norm_topk_prob=True, out=None, ws=None,
                   stream=None, opts: moe_opts | None = None, **opt_kwargs):
    """moe_forward with options; pass a prepared ``opts`` or the keyword arguments of
    ``make_opts`` (router_bias, shared_gate_up, shared_down, shared_gate, residual,
    logits_out, topk_idx_out, topk_w_out, path, stage_events, out_f32, expert_counts_out,
    slot_row_out, wait_limit_us, diag, W_gate_up_fp8, gate_up_scale, W_down_fp8, down_scale).
    With FP8 experts (W_gate_up_fp8 ...), W_gate_up and W_down may be None."""
    if opts is None:
        opts = make_opts(**opt_kwargs)
    fp8 = getattr(opts, "_fp8", (None, None))
    dims = _dims_of(x, W_r, W_gate_up, W_down, k, norm_topk_prob, fp8[0], fp8[1])
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = workspace(dims, opts, device=x.device)
    _check(load().moe_forward_ex(_ptr(x), _ptr(W_r), _ptr(W_gate_up), _ptr(W_down), ctypes.byref(dims),
                                 ctypes.byref(opts), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward_ex")
    return out


def moe_quantize_fp8_rows(W, q=None, scale=None, stream=None):
    """Per-row FP8 E4M3 quantisation of the bf16 matrix W viewed as [rows, W.shape[-1]]:
    -> (q uint8 of W's shape, scale FP32 [rows]).  The format is in the header."""
    _need(W, "W", torch.bfloat16)
    cols = int(W.shape[-1])
    rows = W.numel() // cols if cols else 0
    if q is None:
        q = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=W.device)
    _need(q, "q", torch.uint8)
    _need(scale, "scale", torch.float32)
    _check(load().moe_quantize_fp8_rows(_ptr(W), rows, cols, _ptr(q), _ptr(scale), _stream(stream)),
           "moe_quantize_fp8_rows")
    return q, scale


def moe_forward_noalloc(x, W_r, W_gate_up, W_down, k, norm_topk_prob=True, out=None, stream=None):
    """moe_forward without a workspace argument: for callers that cannot allocate device
    memory, the library uses its own fixed 64 MiB device array (see the header)."""
    dims = _dims_of(x, W_r, W_gate_up, W_down, k, norm_topk_prob)
    if out is None:
        out = torch.empty_like(x)
    _check(load().moe_forward_noalloc(_ptr(x), _ptr(W_r), _ptr(W_gate_up), _ptr(W_down),
                                      ctypes.byref(dims), _ptr(out), _stream(stream)),
           "moe_forward_noalloc")
    return out


def moe_get_device_status(ws, stream=None) -> int:
    return int(load().moe_get_device_status(_ptr(ws), _stream(stream)))


def moe_get_device_status_noalloc(stream=None) -> int:
    return int(load().moe_get_device_status_noalloc(_stream(stream)))


def stage_events(n=6):
    """CUDA events usable as ``stage_events`` (each recorded once so its handle exists)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for ev in evs:
        ev.record()
    return evs
