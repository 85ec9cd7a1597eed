"""ctypes front end of the CPU oracle in ``moe_oracle.c``.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never imports, links or calls it, and it imports
nothing from the product package.

The oracle evaluates the plain definition of a Qwen-family sparse MoE FFN block (pages
"27. Mixture of experts", sections "The router", "The shared expert" and "Dispatch"; and
"Qwen3-VL and Mixture of Experts", section "What a mixture-of-experts layer is") in IEEE
double, one token at a time.  bf16 tensors cross this boundary as their uint16 bit patterns.

Pins: every function here is pinned in ``tests/test_oracle_pins.py`` against values the
pages print, closed forms, library routines on special cases and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            l = ctypes.CDLL(build())
            c_int = ctypes.c_int
            l.oracle_router_logits.argtypes = [_u16p, _u16p, _f32p, c_int, c_int, c_int, _f32p]
            l.oracle_select.argtypes = [_f32p, c_int, c_int, c_int, c_int, _i32p, _f32p]
            l.oracle_route.argtypes = [_u16p, _u16p, _f32p, c_int, c_int, c_int, c_int, c_int,
                                       _f32p, _i32p, _f32p]
            l.oracle_permute.argtypes = [_i32p, c_int, c_int, c_int, c_int, _i32p, _i32p, _i32p,
                                         _i32p, c_int]
            l.oracle_combine_rows.argtypes = [_u16p, _i32p, _f32p, _i32p, c_int, c_int, c_int,
                                              c_int, c_int, c_int, _u16p, _u16p, _u16p, _u16p,
                                              _u16p, c_int, _u16p, _f64p]
            l.oracle_forward_rows.argtypes = [_u16p, _u16p, _f32p, _u16p, _u16p, _i32p, c_int,
                                              c_int, c_int, c_int, c_int, c_int, c_int, _u16p,
                                              _u16p, _u16p, c_int, _u16p, _f64p, _i32p, _f32p,
                                              _f32p]
            l.oracle_loop_dispatch.argtypes = [_u16p, _i32p, _f32p, c_int, c_int, c_int, c_int,
                                               c_int, _u16p, _u16p, _f64p]
            l.oracle_aux_loss.argtypes = [_f32p, _i32p, c_int, c_int, c_int, ctypes.c_double,
                                          ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
            l.oracle_backward.argtypes = [_u16p, _u16p, _f32p, _u16p, _u16p, _u16p, _i32p, c_int, c_int,
                                          c_int, c_int, c_int, c_int, c_int, _f64p, _f64p, _f64p,
                                          _f64p, _f64p, _f64p, _i32p, c_int, _f64p, _f64p]
            l.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            l.oracle_e4m3_value.restype = ctypes.c_double
            l.oracle_quantize_fp8_rows.argtypes = [_u16p, ctypes.c_long, c_int, _u8p, _f32p]
            l.oracle_combine_rows_fp8.argtypes = [_u16p, _i32p, _f32p, _i32p, c_int, c_int, c_int,
                                                  c_int, c_int, c_int, _u8p, _f32p, _u8p, _f32p,
                                                  _u16p, _f64p]
            for name in ("oracle_router_logits", "oracle_select", "oracle_route", "oracle_permute",
                         "oracle_combine_rows", "oracle_forward_rows", "oracle_loop_dispatch",
                         "oracle_quantize_fp8_rows", "oracle_combine_rows_fp8", "oracle_backward"):
                getattr(l, name).restype = ctypes.c_int
            _lib = l
    return _lib


# ------------------------------------------------------------------ marshalling helpers

def as_u16(a) -> np.ndarray:
    """bf16 tensor (torch, CPU) or uint16 array -> contiguous uint16 numpy array of bits."""
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        import torch  # plain CPU torch is used for the bit view only
        a = a.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.uint16)


def _p(a, ptype):
    if a is None:
        return ctypes.cast(None, ptype)
    return a.ctypes.data_as(ptype)


def _f32(a):
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


# ------------------------------------------------------------------ public functions

def router_logits(x, W_r, bias=None):
    """FP32 logits [T, E]: fl32(sum_d x W_r) (+ bias in FP32)."""
    x, W_r, bias = as_u16(x), as_u16(W_r), _f32(bias)
    T, D = x.shape
    E = W_r.shape[0]
    out = np.empty((T, E), np.float32)
    _check(lib().oracle_router_logits(_p(x, _u16p), _p(W_r, _u16p), _p(bias, _f32p), T, D, E,
                                      _p(out, _f32p)), "oracle_router_logits")
    return out


def select(logits, k, norm=True):
    """(idx [T, k] int32, w [T, k] float32) from FP32 logits [T, E]."""
    logits = _f32(logits)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(lib().oracle_select(_p(logits, _f32p), T, E, k, int(bool(norm)), _p(idx, _i32p),
                               _p(w, _f32p)), "oracle_select")
    return idx, w


def route(x, W_r, k, norm=True, bias=None):
    logits = router_logits(x, W_r, bias)
    idx, w = select(logits, k, norm)
    return logits, idx, w


def permute(idx, E, tile_m=1, cap=None):
    """Stable counting sort of the assignments by expert (see moe_oracle.c)."""
    idx = _i32(idx)
    T, k = idx.shape
    if cap is None:
        cap = T * k + E * (tile_m - 1)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_token = np.empty(cap, np.int32)
    slot_row = np.empty(T * k, np.int32)
    _check(lib().oracle_permute(_p(idx, _i32p), T, k, E, tile_m, _p(counts, _i32p),
                                _p(offsets, _i32p), _p(row_token, _i32p), _p(slot_row, _i32p), cap),
           "oracle_permute")
    return counts, offsets, row_token, slot_row


def _chunks(rows, threads):
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    threads = max(1, min(int(threads), len(rows))) if len(rows) else 1
    return np.array_split(rows, threads)


def combine_rows(x, idx, w, rows, W_gu, W_dn, shared_gate_up=None, shared_down=None,
                 shared_gate=None, residual=None, threads=1):
    """y [len(rows), D] (float64) for the given routing of every token."""
    x, W_gu, W_dn = as_u16(x), as_u16(W_gu), as_u16(W_dn)
    sgu, sdn, sg, res = as_u16(shared_gate_up), as_u16(shared_down), as_u16(shared_gate), as_u16(residual)
    idx, w = _i32(idx), _f32(w)
    T, D = x.shape
    k = idx.shape[1]
    E = W_gu.shape[0]
    I = W_gu.shape[1] // 2
    I_s = sgu.shape[0] // 2 if sgu is not None else 0
    parts = _chunks(rows, threads)
    outs = [np.empty((len(p), D), np.float64) for p in parts]

    def run(i):
        p = parts[i]
        _check(lib().oracle_combine_rows(_p(x, _u16p), _p(idx, _i32p), _p(w, _f32p), _p(p, _i32p),
                                         len(p), T, D, E, k, I, _p(W_gu, _u16p), _p(W_dn, _u16p),
                                         _p(sgu, _u16p), _p(sdn, _u16p), _p(sg, _u16p), I_s,
                                         _p(res, _u16p), _p(outs[i], _f64p)), "oracle_combine_rows")

    with ThreadPoolExecutor(max_workers=len(parts)) as ex:
        list(ex.map(run, range(len(parts))))
    return np.concatenate(outs, axis=0) if outs else np.empty((0, D))


def forward_rows(x, W_r, W_gu, W_dn, k, rows, norm=True, bias=None, shared_gate_up=None,
                 shared_down=None, shared_gate=None, residual=None, threads=1):
    """Whole block for the listed rows -> (y [n, D] float64, idx [n, k], w [n, k], logits [n, E])."""
    x, W_r, W_gu, W_dn = as_u16(x), as_u16(W_r), as_u16(W_gu), as_u16(W_dn)
    sgu, sdn, sg, res = as_u16(shared_gate_up), as_u16(shared_down), as_u16(shared_gate), as_u16(residual)
    bias = _f32(bias)
    T, D = x.shape
    E = W_r.shape[0]
    I = W_gu.shape[1] // 2
    I_s = sgu.shape[0] // 2 if sgu is not None else 0
    parts = _chunks(rows, threads)
    res_y = [np.empty((len(p), D), np.float64) for p in parts]
    res_i = [np.empty((len(p), k), np.int32) for p in parts]
    res_w = [np.empty((len(p), k), np.float32) for p in parts]
    res_l = [np.empty((len(p), E), np.float32) for p in parts]

    def run(i):
        p = parts[i]
        _check(lib().oracle_forward_rows(_p(x, _u16p), _p(W_r, _u16p), _p(bias, _f32p),
                                         _p(W_gu, _u16p), _p(W_dn, _u16p), _p(p, _i32p), len(p), T,
                                         D, E, k, I, int(bool(norm)), _p(sgu, _u16p), _p(sdn, _u16p),
                                         _p(sg, _u16p), I_s, _p(res, _u16p), _p(res_y[i], _f64p),
                                         _p(res_i[i], _i32p), _p(res_w[i], _f32p),
                                         _p(res_l[i], _f32p)), "oracle_forward_rows")

    with ThreadPoolExecutor(max_workers=len(parts)) as ex:
        list(ex.map(run, range(len(parts))))
    cat = lambda xs, shape: np.concatenate(xs, axis=0) if xs else np.empty(shape)
    return (cat(res_y, (0, D)), cat(res_i, (0, k)), cat(res_w, (0, k)), cat(res_l, (0, E)))


def loop_dispatch(x, idx, w, W_gu, W_dn):
    """The per-expert gather / run / scatter-add dispatch over all T tokens -> [T, D] float64."""
    x, W_gu, W_dn = as_u16(x), as_u16(W_gu), as_u16(W_dn)
    idx, w = _i32(idx), _f32(w)
    T, D = x.shape
    k = idx.shape[1]
    E = W_gu.shape[0]
    I = W_gu.shape[1] // 2
    y = np.empty((T, D), np.float64)
    _check(lib().oracle_loop_dispatch(_p(x, _u16p), _p(idx, _i32p), _p(w, _f32p), T, D, E, k, I,
                                      _p(W_gu, _u16p), _p(W_dn, _u16p), _p(y, _f64p)),
           "oracle_loop_dispatch")
    return y


def e4m3_value(code: int) -> float:
    """The value of one E4M3 code (NaN for the NaN codes)."""
    return float(lib().oracle_e4m3_value(int(code) & 0xFF))


def quantize_fp8_rows(W):
    """Per-row E4M3 quantisation of W viewed as [rows, W.shape[-1]] -> (q uint8 of W's shape,
    scale float32 [rows])."""
    W = as_u16(W)
    cols = W.shape[-1]
    rows = W.size // cols
    q = np.empty(W.shape, np.uint8)
    scale = np.empty(rows, np.float32)
    _check(lib().oracle_quantize_fp8_rows(_p(W, _u16p), rows, cols, _p(q, _u8p), _p(scale, _f32p)),
           "oracle_quantize_fp8_rows")
    return q, scale


def combine_rows_fp8(x, idx, w, rows, q_gu, s_gu, q_dn, s_dn, residual=None, threads=1):
    """y [len(rows), D] (float64) with FP8 routed experts (weight = scale[row] * value(q))."""
    x, res = as_u16(x), as_u16(residual)
    q_gu = np.ascontiguousarray(np.asarray(q_gu.cpu() if hasattr(q_gu, "cpu") else q_gu), dtype=np.uint8)
    q_dn = np.ascontiguousarray(np.asarray(q_dn.cpu() if hasattr(q_dn, "cpu") else q_dn), dtype=np.uint8)
    s_gu, s_dn = _f32(s_gu), _f32(s_dn)
    idx, w = _i32(idx), _f32(w)
    T, D = x.shape
    k = idx.shape[1]
    E = q_gu.shape[0]
    I = q_gu.shape[1] // 2
    parts = _chunks(rows, threads)
    outs = [np.empty((len(p), D), np.float64) for p in parts]

    def run(i):
        p = parts[i]
        _check(lib().oracle_combine_rows_fp8(_p(x, _u16p), _p(idx, _i32p), _p(w, _f32p), _p(p, _i32p),
                                             len(p), T, D, E, k, I, _p(q_gu, _u8p), _p(s_gu, _f32p),
                                             _p(q_dn, _u8p), _p(s_dn, _f32p), _p(res, _u16p),
                                             _p(outs[i], _f64p)), "oracle_combine_rows_fp8")

    with ThreadPoolExecutor(max_workers=len(parts)) as ex:
        list(ex.map(run, range(len(parts))))
    return np.concatenate(outs, axis=0) if outs else np.empty((0, D))


def aux_loss(logits, idx, alpha=1.0, with_grad=True):
    """Switch balance loss alpha * E * sum_e f_e P_e and (f fixed) its gradient with respect to
    the logits, in double (see oracle_aux_loss).  -> (loss, dlogits [T, E] float64 or None)."""
    lg = _f32(logits)
    ix = _i32(idx)
    T, E = lg.shape
    k = ix.shape[1]
    loss = ctypes.c_double(0.0)
    d = np.zeros((T, E), np.float64) if with_grad else None
    _check(lib().oracle_aux_loss(_p(lg, _f32p), _p(ix, _i32p), T, E, k, float(alpha), ctypes.byref(loss),
                                 d.ctypes.data_as(ctypes.c_void_p) if d is not None else None), "oracle_aux_loss")
    return loss.value, d


def backward(x, W_r, W_gu, W_dn, dy, idx, norm=True, bias=None, residual=False, dlogits_add=None,
             experts=()):
    """Gradients of sum_t dy[t] . y[t] for the given routing idx [T, k] (selection held fixed),
    in double (see oracle_backward).  -> dict with dx [T, D], dW_r [E, D], db [E],
    dlogits [T, E], dw [T, k], and dW_gu [n, 2I, D], dW_dn [n, D, I] for the listed experts."""
    x, W_r, W_gu, W_dn, dy = as_u16(x), as_u16(W_r), as_u16(W_gu), as_u16(W_dn), as_u16(dy)
    bias, ix = _f32(bias), _i32(idx)
    T, D = x.shape
    E, k = W_r.shape[0], ix.shape[1]
    I = W_gu.shape[1] // 2
    ex = np.ascontiguousarray(np.asarray(experts, dtype=np.int32).reshape(-1))
    n = len(ex)
    add = None if dlogits_add is None else np.ascontiguousarray(dlogits_add, dtype=np.float64)
    out = dict(dx=np.empty((T, D)), dW_r=np.empty((E, D)), db=np.empty(E), dlogits=np.empty((T, E)),
               dw=np.empty((T, k)), dW_gu=np.empty((n, 2 * I, D)), dW_dn=np.empty((n, D, I)))
    _check(lib().oracle_backward(_p(x, _u16p), _p(W_r, _u16p), _p(bias, _f32p), _p(W_gu, _u16p),
                                 _p(W_dn, _u16p), _p(dy, _u16p), _p(ix, _i32p), T, D, E, k, I,
                                 int(bool(norm)), int(bool(residual)), _p(add, _f64p),
                                 _p(out["dx"], _f64p), _p(out["dW_r"], _f64p), _p(out["db"], _f64p),
                                 _p(out["dlogits"], _f64p), _p(out["dw"], _f64p), _p(ex, _i32p), n,
                                 _p(out["dW_gu"], _f64p) if n else None,
                                 _p(out["dW_dn"], _f64p) if n else None), "oracle_backward")
    return out


def cpu_threads_available() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
