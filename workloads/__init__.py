"""Seeded synthetic inputs for the 1D deformable convolution forward.

This module is shared by the CUDA path's tests and bench and by the CPU
oracle's tests.  It holds NONE of the method's arithmetic: it only names the
workload shapes and draws random tensors of the stated distributions.  The
output length ``L_out`` that sizes the offset and mask tensors is passed in by
the caller (the five named workloads state it; tests compute it with the
oracle), so no closed form lives here.

Recipe (applies to every workload): one CPU ``torch.Generator`` seeded with
``seed`` (default 0); tensors are drawn in float32 in the fixed order
x, weight, bias, offsets, mask, and cast to bfloat16 (float16) afterwards where the
workload is bf16 (f16).  ``N(0, s)`` means mean 0 and standard deviation ``s``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes, hyper-parameters and input distributions of one synthetic case."""

    name: str
    B: int
    C_in: int
    C_out: int
    K: int
    stride: int
    padding: int
    dilation: int
    groups: int
    offset_groups: int
    L_in: int
    L_out: int                # stated with the workload, not computed here
    dtype: str                # "f32", "bf16" or "f16"
    x_dist: tuple             # ("uniform", lo, hi) | ("normal", std)
    w_dist: tuple             # ("normal", std) | ("kaiming_uniform",) | ("kaiming_normal",)
    bias_dist: Optional[tuple]
    off_dist: tuple
    mask: bool
    unconstrained: bool

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[self.dtype]

    @property
    def fan_in(self) -> int:
        return (self.C_in // self.groups) * self.K

    def flops(self) -> int:
        """Multiply-adds of the contraction, counted as 2 flops each."""
        return 2 * self.B * self.L_out * self.C_out * (self.C_in // self.groups) * self.K

    def algorithmic_bytes(self) -> int:
        """Every tensor counted once: inputs read once, output written once."""
        es = 4 if self.dtype == "f32" else 2
        n = self.B * self.C_in * self.L_in                      # x
        n += self.B * self.offset_groups * self.L_out * self.K  # offsets
        if self.mask:
            n += self.B * self.offset_groups * self.L_out * self.K
        n += self.C_out * (self.C_in // self.groups) * self.K   # weight
        if self.bias_dist is not None:
            n += self.C_out
        n += self.B * self.C_out * self.L_out                   # out
        return n * es

    def with_batch(self, B: int) -> "Workload":
        return dataclasses.replace(self, B=B)


# The five workloads: shapes and distributions as the headline metric states them.
TINY_F32 = Workload(
    name="tiny_f32", B=1, C_in=4, C_out=4, K=3, stride=1, padding=0, dilation=1,
    groups=1, offset_groups=1, L_in=16, L_out=14, dtype="f32",
    x_dist=("uniform", 0.0, 1.0), w_dist=("normal", 0.1), bias_dist=("normal", 0.1),
    off_dist=("uniform", -2.0, 2.0), mask=False, unconstrained=False)

USAGE_F32 = Workload(
    name="usage_f32", B=16, C_in=512, C_out=512, K=16, stride=1, padding=0, dilation=3,
    groups=1, offset_groups=1, L_in=128, L_out=83, dtype="f32",
    x_dist=("uniform", 0.0, 1.0), w_dist=("kaiming_uniform",),
    bias_dist=("uniform", -0.05, 0.05), off_dist=("normal", 1.5), mask=False,
    unconstrained=False)

DEPTHWISE_BF16 = Workload(
    name="depthwise_bf16", B=8, C_in=512, C_out=512, K=3, stride=1, padding=64, dilation=64,
    groups=512, offset_groups=512, L_in=16000, L_out=16000, dtype="bf16",
    x_dist=("normal", 1.0), w_dist=("normal", 0.3), bias_dist=None,
    off_dist=("normal", 4.0), mask=False, unconstrained=True)

MODULATED_BF16 = Workload(
    name="modulated_bf16", B=16, C_in=256, C_out=256, K=5, stride=1, padding=2, dilation=1,
    groups=1, offset_groups=8, L_in=4096, L_out=4096, dtype="bf16",
    x_dist=("normal", 1.0), w_dist=("kaiming_normal",), bias_dist=None,
    off_dist=("uniform", -3.0, 3.0), mask=True, unconstrained=False)

LARGE_BF16 = Workload(
    name="large_bf16", B=32, C_in=1024, C_out=1024, K=9, stride=2, padding=4, dilation=2,
    groups=4, offset_groups=4, L_in=8192, L_out=4092, dtype="bf16",
    x_dist=("normal", 1.0), w_dist=("kaiming_normal",), bias_dist=("normal", 0.02),
    off_dist=("normal", 2.0), mask=False, unconstrained=True)

# PackedDeformConv1d(modulated=True): the dc1d page's example layer (depthwise, one offset
# group per channel, kernel 3, dilation 4, padding "same") at a long-signal size.  Its offsets
# and mask come from the layer's own trunk; off_dist sets the spread of the predicted offsets.
PACKED_MODULATED_BF16 = Workload(
    name="packed_modulated_bf16", B=8, C_in=256, C_out=256, K=3, stride=1, padding=4,
    dilation=4, groups=256, offset_groups=256, L_in=16384, L_out=16384, dtype="bf16",
    x_dist=("normal", 1.0), w_dist=("normal", 0.3), bias_dist=("normal", 0.02),
    off_dist=("normal", 2.0), mask=True, unconstrained=False)

PACKED = {w.name: w for w in (PACKED_MODULATED_BF16,)}

WORKLOADS = {w.name: w for w in (TINY_F32, USAGE_F32, DEPTHWISE_BF16, MODULATED_BF16, LARGE_BF16)}
ORDERED = [TINY_F32, USAGE_F32, DEPTHWISE_BF16, MODULATED_BF16, LARGE_BF16]


def _draw(gen: torch.Generator, shape, dist: tuple, fan_in: int) -> torch.Tensor:
    kind = dist[0]
    if kind == "uniform":
        lo, hi = dist[1], dist[2]
        return torch.rand(shape, generator=gen, dtype=torch.float32) * (hi - lo) + lo
    if kind == "normal":
        return torch.randn(shape, generator=gen, dtype=torch.float32) * dist[1]
    if kind == "kaiming_uniform":   # gain sqrt(2), bound = gain * sqrt(3 / fan_in)
        bound = math.sqrt(6.0 / fan_in)
        return (torch.rand(shape, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound
    if kind == "kaiming_normal":    # std = sqrt(2 / fan_in)
        return torch.randn(shape, generator=gen, dtype=torch.float32) * math.sqrt(2.0 / fan_in)
    if kind == "sigmoid_normal":
        return torch.sigmoid(torch.randn(shape, generator=gen, dtype=torch.float32))
    raise ValueError(f"unknown distribution {dist!r}")


def make_inputs(w: Workload, seed: int = 0) -> dict:
    """Draw the workload's tensors on the CPU.

    Returns a dict with x [B, C_in, L_in], weight [C_out, C_in/groups, K],
    bias [C_out] or None, offsets [B, offset_groups, L_out, K] and mask (same
    shape as offsets) or None, all in the workload's dtype and contiguous.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    x = _draw(gen, (w.B, w.C_in, w.L_in), w.x_dist, w.fan_in)
    weight = _draw(gen, (w.C_out, w.C_in // w.groups, w.K), w.w_dist, w.fan_in)
    bias = _draw(gen, (w.C_out,), w.bias_dist, w.fan_in) if w.bias_dist is not None else None
    offsets = _draw(gen, (w.B, w.offset_groups, w.L_out, w.K), w.off_dist, w.fan_in)
    mask = _draw(gen, offsets.shape, ("sigmoid_normal",), w.fan_in) if w.mask else None
    dt = w.torch_dtype
    out = {"x": x, "weight": weight, "bias": bias, "offsets": offsets, "mask": mask}
    return {k: (v.to(dt).contiguous() if v is not None else None) for k, v in out.items()}


def small_case(seed: int, *, B, C_in, C_out, K, stride, padding, dilation, groups,
               offset_groups, L_in, L_out, dtype="f32", mask=False, bias=True,
               unconstrained=False, off_scale=2.0) -> tuple:
    """A small random case for sweeps of shapes (not one of the named workloads)."""
    w = Workload(
        name="small", B=B, C_in=C_in, C_out=C_out, K=K, stride=stride, padding=padding,
        dilation=dilation, groups=groups, offset_groups=offset_groups, L_in=L_in, L_out=L_out,
        dtype=dtype, x_dist=("normal", 1.0), w_dist=("normal", 0.5),
        bias_dist=("normal", 0.5) if bias else None, off_dist=("normal", off_scale),
        mask=mask, unconstrained=unconstrained)
    return w, make_inputs(w, seed)


def make_packed_inputs(w: Workload, seed: int = 0, modulated: Optional[bool] = None,
                       biases: bool = True) -> dict:
    """Draw PackedDeformConv1d's tensors on the CPU (same generator recipe as make_inputs).

    Order: x [B, C_in, L_in] ~ x_dist; dw_weight [C_in, 1, K] ~ N(0, 1/sqrt(K)); dw_bias
    [C_in] ~ N(0, 0.1); off_weight [G*K, C_in] ~ N(0, s/sqrt(C_in)) with s the std of
    off_dist (so the predicted offsets spread about that much); off_bias [G*K] ~ N(0, 0.1);
    mask_weight [G*K, C_in] ~ N(0, 1.5/sqrt(C_in)) and mask_bias ~ N(0, 0.1) when modulated
    (default: the workload's mask flag); weight and bias as in make_inputs.  Biases are None
    when ``biases`` is False.
    """
    if modulated is None:
        modulated = w.mask
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    J = w.offset_groups * w.K
    s_off = w.off_dist[1] if w.off_dist[0] == "normal" else 1.0

    def normal(shape, std):
        return torch.randn(shape, generator=gen, dtype=torch.float32) * std

    x = _draw(gen, (w.B, w.C_in, w.L_in), w.x_dist, w.fan_in)
    dw_weight = normal((w.C_in, 1, w.K), 1.0 / math.sqrt(w.K))
    dw_bias = normal((w.C_in,), 0.1)
    off_weight = normal((J, w.C_in), s_off / math.sqrt(w.C_in))
    off_bias = normal((J,), 0.1)
    mask_weight = normal((J, w.C_in), 1.5 / math.sqrt(w.C_in)) if modulated else None
    mask_bias = normal((J,), 0.1) if modulated else None
    weight = _draw(gen, (w.C_out, w.C_in // w.groups, w.K), w.w_dist, w.fan_in)
    bias = _draw(gen, (w.C_out,), w.bias_dist, w.fan_in) if w.bias_dist is not None else None
    out = {"x": x, "dw_weight": dw_weight, "dw_bias": dw_bias, "off_weight": off_weight,
           "off_bias": off_bias, "mask_weight": mask_weight, "mask_bias": mask_bias,
           "weight": weight, "bias": bias}
    if not biases:
        for k in ("dw_bias", "off_bias", "mask_bias", "bias"):
            out[k] = None
    dt = w.torch_dtype
    return {k: (v.to(dt).contiguous() if v is not None else None) for k, v in out.items()}


def packed_case(seed: int, *, B, C_in, C_out, K, stride, padding, dilation, groups,
                offset_groups, L_in, L_out, dtype="f32", modulated=True, biases=True,
                off_scale=2.0) -> tuple:
    """A small random PackedDeformConv1d case (not one of the named workloads)."""
    w = Workload(
        name="packed_small", B=B, C_in=C_in, C_out=C_out, K=K, stride=stride, padding=padding,
        dilation=dilation, groups=groups, offset_groups=offset_groups, L_in=L_in, L_out=L_out,
        dtype=dtype, x_dist=("normal", 1.0), w_dist=("normal", 0.5),
        bias_dist=("normal", 0.5) if biases else None, off_dist=("normal", off_scale),
        mask=modulated, unconstrained=False)
    return w, make_packed_inputs(w, seed, modulated, biases)
