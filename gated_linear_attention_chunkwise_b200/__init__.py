"""DiG gated-linear-attention hot path on B200 -- thin Python binding.

Every function here only checks shapes/dtypes (for readable errors), picks the
caller's current CUDA stream and forwards raw device pointers to the C ABI of
`libdig_gla.so` (declared in include/dig_gla.h).  All computation happens in
the library's sm_100a kernels; there is no CPU or PyTorch fallback, and
importing this package fails if the library has not been built
(`python gated_linear_attention_chunkwise_b200/build.py`).

Names follow the C ABI: gla_fwd, gla_fwd_glogit, gla_fwd_f32, gla_bwd, gla_bwd_f32, gla_norm_fwd,
gla_norm_fwd_f32, srem_reorient, dwconv3x3,
device_status (dig_gla_device_status), status_string (dig_gla_status_string).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["gla_fwd", "gla_fwd_glogit", "gla_fwd_f32", "gla_bwd", "gla_bwd_f32", "gla_norm_fwd", "gla_norm_fwd_f32", "srem_reorient", "dwconv3x3", "device_status", "status_string",
           "GlaError", "lib", "LIB_PATH", "DIR_L2R", "DIR_R2L", "DIR_T2B", "DIR_B2T"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdig_gla.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python gated_linear_attention_chunkwise_b200/build.py`"
                      " (nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _u = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
_lib.gla_fwd.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 7 + [_vp, _u]
_lib.gla_fwd_f32.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 7 + [_vp, _u]
_lib.gla_bwd.argtypes = [_vp] * 5 + [_i] * 7 + [_vp] * 4 + [_u]
_lib.gla_bwd_f32.argtypes = [_vp] * 5 + [_i] * 7 + [_vp] * 4 + [_u]
_lib.gla_fwd_glogit.argtypes = [_vp] * 4 + [_i] * 7 + [ctypes.c_float, _vp, _u]
_lib.gla_norm_fwd.argtypes = [_vp] * 3 + [_i] * 7 + [ctypes.c_float, _vp, _u]
_lib.gla_norm_fwd_f32.argtypes = [_vp] * 3 + [_i] * 7 + [ctypes.c_float, _vp, _u]
_lib.srem_reorient.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _i, _vp, _u]
_lib.dwconv3x3.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _u]
_lib.dig_gla_device_status.argtypes = [_u]
_lib.dig_gla_status_string.argtypes = [_i]
_lib.dig_gla_status_string.restype = ctypes.c_char_p
_lib.dig_gla_release.argtypes = []
_lib.dig_gla_release.restype = None
_lib.dig_gla_test_skip_items.argtypes = [_i]
_lib.dig_gla_test_skip_items.restype = None
for _fn in (_lib.gla_fwd, _lib.gla_fwd_glogit, _lib.gla_fwd_f32, _lib.gla_bwd, _lib.gla_bwd_f32, _lib.gla_norm_fwd, _lib.gla_norm_fwd_f32,
            _lib.srem_reorient, _lib.dwconv3x3, _lib.dig_gla_device_status):
    _fn.restype = ctypes.c_int

DIR_L2R, DIR_R2L, DIR_T2B, DIR_B2T = 0, 1, 2, 3
_BF16, _F32 = 0, 1


def lib() -> ctypes.CDLL:
    """The loaded C library (for callers that pass raw pointers themselves)."""
    return _lib


class GlaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return _lib.dig_gla_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != 0:
        raise GlaError(fn, rc)


def _stream_handle(dev: torch.device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, dev: torch.device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != dev or t.device.type != "cuda":
        raise ValueError(f"{name} must be on {dev} (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _gla(fn_name: str, q, k, v, log_alpha, Hgrid, Wgrid, direction, out, stream, dtype):
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dtype, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    if q.dim() != 4 or k.shape != q.shape or log_alpha.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q, k, log_alpha [B,T,H,dk] and v [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if T != Hgrid * Wgrid:
        raise ValueError(f"T={T} does not match the grid {Hgrid}x{Wgrid}")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dtype, device=dev)
    else:
        _need(out, "out", dtype, dev)
        if tuple(out.shape) != (B, T, H, dv):
            raise ValueError("out must be [B,T,H,dv]")
    with torch.cuda.device(dev):
        rc = getattr(_lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), log_alpha.data_ptr(), B, H, Hgrid,
                                    Wgrid, dk, dv, int(direction), out.data_ptr(), _stream_handle(dev, stream))
    _check(fn_name, rc)
    return out


def gla_fwd(q, k, v, log_alpha, Hgrid: int, Wgrid: int, direction: int, out=None, stream=None):
    """bf16 GLA forward (see include/dig_gla.h, gla_fwd).  Returns `out` [B,T,H,dv] bf16."""
    return _gla("gla_fwd", q, k, v, log_alpha, Hgrid, Wgrid, direction, out, stream, torch.bfloat16)


def gla_fwd_glogit(q, k, v, g, Hgrid: int, Wgrid: int, direction: int, gate_norm: float = 16.0, out=None,
                   stream=None):
    """bf16 GLA forward with bf16 gate logits g (log_alpha = logsigmoid(g) / gate_norm in
    the kernel; see include/dig_gla.h, gla_fwd_glogit).  Returns `out` [B,T,H,dv] bf16."""
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g")):
        _need(t, n, torch.bfloat16, dev)
    if q.dim() != 4 or k.shape != q.shape or g.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q, k, g [B,T,H,dk] and v [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if T != Hgrid * Wgrid:
        raise ValueError(f"T={T} does not match the grid {Hgrid}x{Wgrid}")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    else:
        _need(out, "out", torch.bfloat16, dev)
    with torch.cuda.device(dev):
        rc = _lib.gla_fwd_glogit(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), B, H, Hgrid, Wgrid, dk, dv,
                                 int(direction), float(gate_norm), out.data_ptr(), _stream_handle(dev, stream))
    _check("gla_fwd_glogit", rc)
    return out


def gla_fwd_f32(q, k, v, log_alpha, Hgrid: int, Wgrid: int, direction: int, out=None, stream=None):
    """fp32 GLA forward (see include/dig_gla.h, gla_fwd_f32).  Returns `out` [B,T,H,dv] fp32."""
    return _gla("gla_fwd_f32", q, k, v, log_alpha, Hgrid, Wgrid, direction, out, stream, torch.float32)


def _bwd(fn_name: str, q, k, v, log_alpha, dout, Hgrid, Wgrid, direction, stream, dtype):
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, dtype, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    if q.dim() != 4 or k.shape != q.shape or log_alpha.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q, k, log_alpha [B,T,H,dk] and v [B,T,H,dv]")
    if dout.shape != v.shape:
        raise ValueError("dout must be [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if T != Hgrid * Wgrid:
        raise ValueError(f"T={T} does not match the grid {Hgrid}x{Wgrid}")
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty_like(log_alpha)
    with torch.cuda.device(dev):
        rc = getattr(_lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), log_alpha.data_ptr(), dout.data_ptr(),
                                    B, H, Hgrid, Wgrid, dk, dv, int(direction), dq.data_ptr(), dk_.data_ptr(),
                                    dv_.data_ptr(), dla.data_ptr(), _stream_handle(dev, stream))
    _check(fn_name, rc)
    return dq, dk_, dv_, dla


def gla_bwd(q, k, v, log_alpha, dout, Hgrid: int, Wgrid: int, direction: int, stream=None):
    """bf16 GLA backward (see include/dig_gla.h, gla_bwd): the gradients of sum(dout * out)
    for out = gla_fwd(q, k, v, log_alpha, ...).  Returns (dq, dk, dv) bf16 and dlog_alpha fp32."""
    return _bwd("gla_bwd", q, k, v, log_alpha, dout, Hgrid, Wgrid, direction, stream, torch.bfloat16)


def gla_bwd_f32(q, k, v, log_alpha, dout, Hgrid: int, Wgrid: int, direction: int, stream=None):
    """fp32 GLA backward (see include/dig_gla.h, gla_bwd_f32).  Returns (dq, dk, dv, dlog_alpha) fp32."""
    return _bwd("gla_bwd_f32", q, k, v, log_alpha, dout, Hgrid, Wgrid, direction, stream, torch.float32)


def _norm(fn_name, q, k, v, Hgrid, Wgrid, direction, eps, out, stream, dtype):
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dtype, dev)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q, k [B,T,H,dk] and v [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if T != Hgrid * Wgrid:
        raise ValueError(f"T={T} does not match the grid {Hgrid}x{Wgrid}")
    if out is None:
        out = torch.empty_like(v)
    else:
        _need(out, "out", dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must be [B,T,H,dv]")
    with torch.cuda.device(dev):
        rc = getattr(_lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, Hgrid, Wgrid, dk, dv,
                                    int(direction), float(eps), out.data_ptr(), _stream_handle(dev, stream))
    _check(fn_name, rc)
    return out


def gla_norm_fwd(q, k, v, Hgrid: int, Wgrid: int, direction: int, eps: float = 1e-6, out=None, stream=None):
    """The draft's normalised GLA, bf16 (see include/dig_gla.h, gla_norm_fwd)."""
    return _norm("gla_norm_fwd", q, k, v, Hgrid, Wgrid, direction, eps, out, stream, torch.bfloat16)


def gla_norm_fwd_f32(q, k, v, Hgrid: int, Wgrid: int, direction: int, eps: float = 1e-6, out=None, stream=None):
    """The draft's normalised GLA, fp32 (see include/dig_gla.h, gla_norm_fwd_f32)."""
    return _norm("gla_norm_fwd_f32", q, k, v, Hgrid, Wgrid, direction, eps, out, stream, torch.float32)


def _grid_dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return _BF16
    if x.dtype == torch.float32:
        return _F32
    raise TypeError("grid tensors must be bf16 or fp32")


def srem_reorient(x, direction: int, inverse: int, Hgrid: int, Wgrid: int, out=None, stream=None):
    """Row gather into (inverse=0) or out of (inverse=1) the scan order.  x: [B, T, C] or [B, Hg, Wg, C]."""
    dt = _grid_dtype(x)
    _need(x, "x", x.dtype, x.device)
    B = x.shape[0]
    C = x.shape[-1]
    if x.numel() != B * Hgrid * Wgrid * C:
        raise ValueError("x must hold B x Hgrid x Wgrid x C elements")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", x.dtype, x.device)
        if out.numel() != x.numel():
            raise ValueError("out must match x")
    with torch.cuda.device(x.device):
        rc = _lib.srem_reorient(x.data_ptr(), int(direction), int(inverse), B, Hgrid, Wgrid, C, dt, out.data_ptr(),
                                _stream_handle(x.device, stream))
    _check("srem_reorient", rc)
    return out


def dwconv3x3(x, w, out=None, stream=None):
    """Depthwise 3x3 conv, zero padding.  x: [B, Hg, Wg, C] bf16/fp32 channels-last; w: [C, 3, 3] fp32."""
    dt = _grid_dtype(x)
    _need(x, "x", x.dtype, x.device)
    _need(w, "w", torch.float32, x.device)
    if x.dim() != 4 or tuple(w.shape) != (x.shape[3], 3, 3):
        raise ValueError("expected x [B,Hg,Wg,C] and w [C,3,3]")
    B, Hg, Wg, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", x.dtype, x.device)
        if out.shape != x.shape:
            raise ValueError("out must match x")
    with torch.cuda.device(x.device):
        rc = _lib.dwconv3x3(x.data_ptr(), w.data_ptr(), B, Hg, Wg, C, dt, out.data_ptr(),
                            _stream_handle(x.device, stream))
    _check("dwconv3x3", rc)
    return out


def skip_items_for_test(n: int) -> None:
    """Test hook: the next gla_fwd call leaves out its first n work items, so the
    look-back waits that need them run out (device status GLA_ERR_TIMEOUT afterwards,
    output unspecified).  n <= 0 clears it."""
    _lib.dig_gla_test_skip_items(int(n))


def device_status(stream=None, device=None) -> int:
    """Synchronise the stream, then return and clear the device status word (0 = GLA_OK)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(_lib.dig_gla_device_status(_stream_handle(dev, stream)))
