"""Seeded synthetic inputs for the DiG GLA hot path.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic (no recurrence, no scan order, no convolution).  Both the
CPU oracle's tests and the CUDA path's tests/bench draw their inputs from here,
so the two sides always see bit-identical values.

Workloads follow the DiG paper's resolution/patch arithmetic (DiG paper notes,
"整体框架": VAE downsamples 8x, patch size 2, so a grid of (res/16)^2 tokens) and
the five synthetic configurations of the GLA path:

  c1  GLA only, fp32:      B=2, H=6,  16x16  (T=256),   d=64, g~N(0,1),  dir 0
  c2  DiG-S/2 @ 512:       B=8, H=6,  32x32  (T=1024),  d=64, g~N(0,1),  dirs 0-3, conv C=384
  c3  DiG-B/2 @ 1024:      B=4, H=12, 64x64  (T=4096),  d=64, g~N(2,1),  dirs 0-3, conv C=768
  c4  DiG-XL/2 @ 1792:     B=2, H=16, 112x112(T=12544), d=72, g~N(0,1),  dirs 0-3, conv C=1152
  c5  DiG-XL/2 @ 2048:     B=1, H=16, 128x128(T=16384), d=72, g~N(-1,1), 28 layers

Values: q, k, v ~ N(0,1) * 1/sqrt(d); log_alpha = logsigmoid(g)/16 per key
channel per token; conv weight = identity 3x3 kernel + 0.01*N(0,1).
Draw order with one CPU torch.Generator seeded by `seed`: q, k, v, g, then w.
q/k/v are drawn in fp32 and cast to bf16 for the bf16 workloads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hgrid: int
    Wgrid: int
    dk: int
    dv: int
    dtype: str          # "f32" or "bf16" for q/k/v/out (log_alpha is always fp32)
    g_mean: float       # mean of the gate pre-activation g
    dirs: tuple         # scan directions exercised
    layers: int = 1     # layers in the stack (c5); dir of layer l is l % 4

    @property
    def T(self) -> int:
        return self.Hgrid * self.Wgrid

    @property
    def C(self) -> int:
        """Channel count of the conv / reorient input (heads x value width)."""
        return self.H * self.dv

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H


WORKLOADS = {
    "c1": Workload("c1_gla_f32_T256", 2, 6, 16, 16, 64, 64, "f32", 0.0, (0,)),
    "c2": Workload("c2_digS2_res512_T1024", 8, 6, 32, 32, 64, 64, "bf16", 0.0, (0, 1, 2, 3)),
    "c3": Workload("c3_digB2_res1024_T4096", 4, 12, 64, 64, 64, 64, "bf16", 2.0, (0, 1, 2, 3)),
    "c4": Workload("c4_digXL2_res1792_T12544", 2, 16, 112, 112, 72, 72, "bf16", 0.0, (0, 1, 2, 3)),
    "c5": Workload("c5_digXL2_res2048_T16384_28L", 1, 16, 128, 128, 72, 72, "bf16", -1.0,
                   (0, 1, 2, 3), layers=28),
}


def custom(B, H, Hgrid, Wgrid, dk, dv, dtype="bf16", g_mean=0.0, name="custom"):
    return Workload(name, B, H, Hgrid, Wgrid, dk, dv, dtype, g_mean, (0, 1, 2, 3))


def gla_inputs(w: Workload, seed: int = 0, qkv_scale: float | None = None,
               g_mean: float | None = None, g_std: float = 1.0):
    """Draw (q, k, v, log_alpha) on the CPU.

    Layouts: q, k, log_alpha are [B][T][H][dk]; v is [B][T][H][dv] (token-major,
    heads interleaved, as a fused q/k/v projection writes them).  q/k/v have the
    workload's dtype, log_alpha is fp32.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    scale = (1.0 / math.sqrt(w.dk)) if qkv_scale is None else qkv_scale
    gm = w.g_mean if g_mean is None else g_mean
    shp_k = (w.B, w.T, w.H, w.dk)
    shp_v = (w.B, w.T, w.H, w.dv)
    q = torch.randn(shp_k, generator=gen, dtype=torch.float32) * scale
    k = torch.randn(shp_k, generator=gen, dtype=torch.float32) * scale
    v = torch.randn(shp_v, generator=gen, dtype=torch.float32) * scale
    g = torch.randn(shp_k, generator=gen, dtype=torch.float32) * g_std + gm
    log_alpha = torch.nn.functional.logsigmoid(g) / 16.0
    if w.dtype == "bf16":
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    return q.contiguous(), k.contiguous(), v.contiguous(), log_alpha.contiguous()


def conv_weight(C: int, seed: int = 0, noise: float = 0.01):
    """Depthwise 3x3 weight [C][3][3] fp32: identity kernel (centre 1) + noise*N(0,1).

    Drawn from its own generator stream (seed + 1_000_003) so that it does not
    depend on the GLA input sizes.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + 1_000_003)
    w = torch.randn((C, 3, 3), generator=gen, dtype=torch.float32) * noise
    w[:, 1, 1] += 1.0
    return w.contiguous()


def grid_tensor(B: int, Hgrid: int, Wgrid: int, C: int, dtype=torch.bfloat16, seed: int = 0):
    """A channels-last token grid [B][Hgrid][Wgrid][C] of N(0,1) values."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + 2_000_003)
    x = torch.randn((B, Hgrid, Wgrid, C), generator=gen, dtype=torch.float32)
    return x.to(dtype).contiguous()


def gla_inputs_device(w: Workload, seed: int, device, qkv_scale: float | None = None):
    """The same recipe as gla_inputs, drawn on `device` from a device generator seeded
    by `seed` (a different random stream from the CPU one, so the values differ from
    gla_inputs'): for timing many fresh layers without a host round trip, never for
    parity checks."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    scale = (1.0 / math.sqrt(w.dk)) if qkv_scale is None else qkv_scale
    shp_k = (w.B, w.T, w.H, w.dk)
    shp_v = (w.B, w.T, w.H, w.dv)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = (torch.randn(shp_k, generator=gen, dtype=torch.float32, device=device) * scale).to(dt)
    k = (torch.randn(shp_k, generator=gen, dtype=torch.float32, device=device) * scale).to(dt)
    v = (torch.randn(shp_v, generator=gen, dtype=torch.float32, device=device) * scale).to(dt)
    g = torch.randn(shp_k, generator=gen, dtype=torch.float32, device=device) + w.g_mean
    log_alpha = torch.nn.functional.logsigmoid(g) / 16.0
    return q.contiguous(), k.contiguous(), v.contiguous(), log_alpha.contiguous()


def conv_weight_device(C: int, seed: int, device, noise: float = 0.01):
    """conv_weight's recipe drawn on `device` (timing only)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) + 1_000_003)
    w = torch.randn((C, 3, 3), generator=gen, dtype=torch.float32, device=device) * noise
    w[:, 1, 1] += 1.0
    return w.contiguous()


def gla_dout(w: Workload, seed: int = 0, scale: float | None = None):
    """An upstream gradient d out [B][T][H][dv] for the GLA backward: N(0,1) * 1/sqrt(dv)
    in the workload's dtype, from its own generator stream (seed + 3_000_003) so that it
    does not change the forward inputs of the same seed."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + 3_000_003)
    s = (1.0 / math.sqrt(w.dv)) if scale is None else scale
    d = torch.randn((w.B, w.T, w.H, w.dv), generator=gen, dtype=torch.float32) * s
    if w.dtype == "bf16":
        d = d.to(torch.bfloat16)
    return d.contiguous()


def gla_inputs_glogit(w: Workload, seed: int = 0):
    """(q, k, v, g) with the same draws as gla_inputs (g before its logsigmoid), g cast to
    bf16: the gate-logit form of the same workload (log_alpha = logsigmoid(g) / 16 of the
    bf16 g)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    scale = 1.0 / math.sqrt(w.dk)
    shp_k = (w.B, w.T, w.H, w.dk)
    shp_v = (w.B, w.T, w.H, w.dv)
    q = torch.randn(shp_k, generator=gen, dtype=torch.float32) * scale
    k = torch.randn(shp_k, generator=gen, dtype=torch.float32) * scale
    v = torch.randn(shp_v, generator=gen, dtype=torch.float32) * scale
    g = torch.randn(shp_k, generator=gen, dtype=torch.float32) + w.g_mean
    return tuple(t.to(torch.bfloat16).contiguous() for t in (q, k, v, g))
