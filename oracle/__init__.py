"""CPU fp64 oracle for the DiG GLA hot path -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this package.  The product path (the CUDA library and its Python
binding) never imports it, and it imports nothing from the product.

The arithmetic lives in `dig_oracle.c` (plain C, fp64); this module only builds
that file with gcc and marshals numpy arrays through ctypes.  Every input is
widened to fp64 exactly (bf16 and fp32 values are representable in fp64), so the
oracle sees the very values the GPU receives.

Functions and the passages they follow (see the C file for the full statement):
  scan_order       DiG notes, SREM: four scan orders by transposing / flipping
                   the 2D token grid.
  gla_fwd          the GLA recurrence S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
                   o_t = q_t S_t over the scan order, zero initial state, update
                   before read (diffusers draft "gated_linear_attention").
  gla_fwd_glogit   the forward with the gate given as logits g:
                   log_alpha = logsigmoid(g) / gate_norm (the configurations' gate).
  gla_bwd          the exact gradient of that recurrence (dq, dk, dv, dlog_alpha
                   for a given d out), as reverse-mode differentiation of its steps
                   in reverse scan order (DiG notes, training like DiT).
  gla_norm_fwd     the diffusers draft's normalised variant (page 4,
                   "gated_linear_attention"): elu+1 features, sigmoid(q*k) gate,
                   gated denominator, output divided by max(denominator, eps).
  dwconv3x3        DiG notes, SREM / DiG Block step (4): 3x3 depthwise conv on
                   the 2D token grid, zero padding.
  reorient         DiG notes, SREM: the O(T) transpose + flip as a row gather.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dig_oracle.c")
_LIB = os.path.join(_HERE, "libdig_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile dig_oracle.c into libdig_oracle.so (gcc, -O2, no fast-math)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                   "-ffp-contract=off", "-pthread", _SRC, "-o", tmp, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        c_int, c_i64 = ctypes.c_int, ctypes.c_int64
        lib.oracle_scan_order.argtypes = [c_int, c_int, c_int, i64p]
        lib.oracle_gla_fwd.argtypes = [dp, dp, dp, dp] + [c_int] * 7 + [dp, c_int]
        lib.oracle_gla_fwd_heads.argtypes = [dp, dp, dp, dp] + [c_int] * 7 + [dp, c_int, c_i64, c_i64]
        lib.oracle_gla_fwd_planted.argtypes = [dp, dp, dp, dp] + [c_int] * 7 + [dp, c_int]
        lib.oracle_gla_bwd.argtypes = [dp] * 5 + [c_int] * 7 + [dp] * 4 + [c_int, c_i64, c_i64]
        lib.oracle_gla_bwd_planted.argtypes = [dp] * 5 + [c_int] * 7 + [dp] * 4 + [c_int]
        lib.oracle_gla_bwd.restype = c_int
        lib.oracle_gla_bwd_planted.restype = c_int
        lib.oracle_gla_fwd_glogit.argtypes = [dp] * 4 + [c_int] * 7 + [ctypes.c_double, dp, c_int]
        lib.oracle_gla_fwd_glogit.restype = c_int
        lib.oracle_gla_norm_fwd.argtypes = [dp] * 3 + [c_int] * 7 + [ctypes.c_double, dp, c_int]
        lib.oracle_gla_norm_fwd_planted.argtypes = [dp] * 3 + [c_int] * 7 + [ctypes.c_double, dp, c_int]
        lib.oracle_gla_norm_fwd.restype = c_int
        lib.oracle_gla_norm_fwd_planted.restype = c_int
        lib.oracle_dwconv3x3.argtypes = [dp, dp, c_int, c_int, c_int, c_int, dp, c_int]
        lib.oracle_reorient.argtypes = [ctypes.c_void_p, c_int, c_int, c_int, c_int, c_int, c_i64,
                                        ctypes.c_void_p]
        lib.oracle_hardware_threads.argtypes = []
        for fn in (lib.oracle_scan_order, lib.oracle_gla_fwd, lib.oracle_gla_fwd_heads,
                   lib.oracle_gla_fwd_planted, lib.oracle_dwconv3x3, lib.oracle_reorient,
                   lib.oracle_hardware_threads):
            fn.restype = c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Widen a numpy array or torch tensor (fp32/bf16/fp64) to contiguous fp64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")
    return rc


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def scan_order(direction: int, Hgrid: int, Wgrid: int) -> np.ndarray:
    """order[p] = raster token id visited at scan position p."""
    out = np.empty(Hgrid * Wgrid, dtype=np.int64)
    _check(_load().oracle_scan_order(direction, Hgrid, Wgrid,
                                     out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))), "scan_order")
    return out


def gla_fwd(q, k, v, log_alpha, Hgrid: int, Wgrid: int, direction: int, nthreads: int = 0,
            heads: tuple | None = None, planted: int = 0, return_threads: bool = False):
    """fp64 GLA forward.  q, k, log_alpha: [B,T,H,dk]; v: [B,T,H,dv] -> out [B,T,H,dv] fp64.

    heads=(begin, end) restricts the work to flattened heads b*H+h in [begin, end)
    (other outputs stay zero).  planted != 0 runs a deliberately wrong variant.
    """
    q, k, v, la = _f64(q), _f64(k), _f64(v), _f64(log_alpha)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    assert T == Hgrid * Wgrid and k.shape == q.shape and la.shape == q.shape and v.shape[:3] == q.shape[:3]
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    lib = _load()
    args = (_dp(q), _dp(k), _dp(v), _dp(la), B, H, Hgrid, Wgrid, dk, dv, direction, _dp(out))
    if planted:
        rc = _check(lib.oracle_gla_fwd_planted(*args, planted), "gla_fwd_planted")
    elif heads is not None:
        rc = _check(lib.oracle_gla_fwd_heads(*args, nthreads, int(heads[0]), int(heads[1])), "gla_fwd")
    else:
        rc = _check(lib.oracle_gla_fwd(*args, nthreads), "gla_fwd")
    return (out, rc) if return_threads else out


def gla_fwd_glogit(q, k, v, g, Hgrid: int, Wgrid: int, direction: int, gate_norm: float = 16.0,
                   nthreads: int = 0) -> np.ndarray:
    """fp64 forward with gate logits g [B,T,H,dk]: log_alpha = logsigmoid(g) / gate_norm."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    assert T == Hgrid * Wgrid and k.shape == q.shape and g.shape == q.shape and v.shape[:3] == q.shape[:3]
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    _check(_load().oracle_gla_fwd_glogit(_dp(q), _dp(k), _dp(v), _dp(g), B, H, Hgrid, Wgrid, dk, dv, direction,
                                         float(gate_norm), _dp(out), nthreads), "gla_fwd_glogit")
    return out


def gla_bwd(q, k, v, log_alpha, dout, Hgrid: int, Wgrid: int, direction: int, nthreads: int = 0,
            heads: tuple | None = None, planted: int = 0):
    """fp64 GLA backward: the gradients (dq, dk, dv, dlog_alpha) of sum(dout * out),
    out = gla_fwd(q, k, v, log_alpha, ...).  Shapes as gla_fwd; dout is [B,T,H,dv].

    heads=(begin, end) restricts the work to flattened heads b*H+h in [begin, end)
    (other gradients stay zero); each worker holds one head's T forward states.
    planted != 0 runs a deliberately wrong variant.
    """
    q, k, v, la, do = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(dout)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    assert T == Hgrid * Wgrid and k.shape == q.shape and la.shape == q.shape and v.shape[:3] == q.shape[:3]
    assert do.shape == v.shape
    gq, gk, gv, gl = (np.zeros(a.shape, dtype=np.float64) for a in (q, k, v, la))
    lib = _load()
    args = (_dp(q), _dp(k), _dp(v), _dp(la), _dp(do), B, H, Hgrid, Wgrid, dk, dv, direction,
            _dp(gq), _dp(gk), _dp(gv), _dp(gl))
    if planted:
        _check(lib.oracle_gla_bwd_planted(*args, planted), "gla_bwd_planted")
    else:
        lo, hi = (0, -1) if heads is None else (int(heads[0]), int(heads[1]))
        _check(lib.oracle_gla_bwd(*args, nthreads, lo, hi), "gla_bwd")
    return gq, gk, gv, gl


def gla_norm_fwd(q, k, v, Hgrid: int, Wgrid: int, direction: int, eps: float = 1e-6, nthreads: int = 0,
                 planted: int = 0) -> np.ndarray:
    """fp64 normalised variant.  q, k: [B,T,H,dk]; v: [B,T,H,dv] -> out [B,T,H,dv]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    assert T == Hgrid * Wgrid and k.shape == q.shape and v.shape[:3] == q.shape[:3]
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    lib = _load()
    args = (_dp(q), _dp(k), _dp(v), B, H, Hgrid, Wgrid, dk, dv, direction, float(eps), _dp(out))
    if planted:
        _check(lib.oracle_gla_norm_fwd_planted(*args, planted), "gla_norm_fwd_planted")
    else:
        _check(lib.oracle_gla_norm_fwd(*args, nthreads), "gla_norm_fwd")
    return out


def dwconv3x3(x, w, nthreads: int = 0) -> np.ndarray:
    """fp64 depthwise 3x3 conv.  x: [B,Hg,Wg,C] channels-last; w: [C,3,3]."""
    x, w = _f64(x), _f64(w)
    B, Hg, Wg, C = x.shape
    assert w.shape == (C, 3, 3)
    y = np.zeros_like(x)
    _check(_load().oracle_dwconv3x3(_dp(x), _dp(w), B, Hg, Wg, C, _dp(y), nthreads), "dwconv3x3")
    return y


def reorient(x: np.ndarray, direction: int, inverse: int, Hgrid: int, Wgrid: int) -> np.ndarray:
    """Byte-exact row gather.  x: [B, T, ...] any dtype (numpy); returns the same dtype."""
    x = np.ascontiguousarray(x)
    B = x.shape[0]
    T = Hgrid * Wgrid
    assert x.shape[1] == T
    row_bytes = x.nbytes // (B * T)
    y = np.empty_like(x)
    _check(_load().oracle_reorient(x.ctypes.data, direction, inverse, B, Hgrid, Wgrid, row_bytes,
                                   y.ctypes.data), "reorient")
    return y
