"""Pins of the oracle's backward (test infrastructure, CPU only).

The backward is the derivative of the forward (the "dc1d (DeformConv1d)" page trains the
layer through autograd and checks the offset gradient against a finite difference in its
demo notebook).  Two independent references pin it here:

- central finite differences of the oracle's FORWARD, for every element of every input,
  on inputs where the difference is exact: values on a bf16 grid and a step of 2^-6 (so
  x +- h and pos +- h are exact in float32), offsets whose fractional part lies in
  [0.25, 0.75] (so pos +- h stays inside one unit cell, where the forward is linear, and
  never crosses a clamp bound); the forward is linear in x, weight, mask and bias, and
  piecewise linear in the offsets, so the central difference equals the derivative up to
  float64 rounding;
- torch's float64 conv1d autograd, for zero offsets and no mask (the forward is then a
  plain conv1d).
Planted mistakes in copies of the backward (below) must each fail one of these pins.
"""
import copy
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import build as obuild

H = 2.0 ** -6

# B, C_in, C_out, K, L_in, stride, padding, dilation, groups, offset_groups, mask, unconstrained
CASES = [
    (2, 4, 6, 3, 10, 1, 1, 1, 2, 2, True, False),
    (1, 4, 4, 3, 12, 2, 2, 2, 1, 1, False, True),
    (2, 2, 4, 4, 9, 1, 0, 1, 2, 1, True, True),
    (1, 6, 3, 2, 7, 1, 1, 3, 3, 3, True, False),
    (2, 4, 4, 4, 11, 1, (1, 2), 1, 2, 2, True, False),   # "same" with d(K-1) odd
]
IDS = ["g2_og2_mask_constrained", "strided_dilated_unc", "k4_mask_unc", "depthwise_like_dil3",
       "same_padding_asymmetric"]


def _bf16_grid(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def make(case, seed=0):
    B, Ci, Co, K, L, s, p, d, G, og, mask, unc = case
    rng = np.random.default_rng(seed)
    L_out = oracle.out_length(L, K, s, p, d)
    ints = rng.integers(-2, 3, size=(B, og, L_out, K))
    frac = rng.integers(64, 193, size=(B, og, L_out, K)) / 256.0   # [0.25, 0.75], 2^-8 grid
    t = {
        "x": _bf16_grid(rng.normal(size=(B, Ci, L))),
        "offsets": (ints + frac).astype(np.float32),
        "mask": _bf16_grid(rng.uniform(0.2, 1.0, size=(B, og, L_out, K))) if mask else None,
        "weight": _bf16_grid(rng.normal(size=(Co, Ci // G, K))),
        "bias": _bf16_grid(rng.normal(size=(Co,))),
        "gout": _bf16_grid(rng.normal(size=(B, Co, L_out))),
    }
    return t, (s, p, d, G, og, unc)


def loss(o, t, args):
    s, p, d, G, og, unc = args
    y = o.forward(t["x"], t["offsets"], t["mask"], t["weight"], t["bias"], s, p, d, G, og, unc)
    return float(np.sum(t["gout"].astype(np.float64) * y))


def fd_grad(o, t, args, key):
    """Central difference of the loss for every element of input ``key``."""
    base = t[key]
    g = np.zeros(base.shape, np.float64)
    for idx in np.ndindex(base.shape):
        tp, tm = copy.copy(t), copy.copy(t)
        tp[key] = base.copy()
        tm[key] = base.copy()
        tp[key][idx] += np.float32(H)
        tm[key][idx] -= np.float32(H)
        g[idx] = (loss(o, tp, args) - loss(o, tm, args)) / (2 * H)
    return g


def backward(o, t, args):
    s, p, d, G, og, unc = args
    return o.backward(t["x"], t["offsets"], t["mask"], t["weight"], t["gout"], s, p, d, G, og,
                      unc)


def pin_finite_differences(o, case):
    t, args = make(case)
    g = backward(o, t, args)
    pairs = [("x", "grad_x"), ("offsets", "grad_offsets"), ("weight", "grad_weight"),
             ("bias", "grad_bias")]
    if t["mask"] is not None:
        pairs.append(("mask", "grad_mask"))
    for key, gkey in pairs:
        ref = fd_grad(o, t, args, key)
        scale = max(1.0, float(np.abs(ref).max()))
        err = float(np.abs(g[gkey] - ref).max())
        assert err <= 1e-9 * scale, (key, err, scale)


def pin_conv1d_autograd(o, case):
    """Zero offsets and no mask: the forward is conv1d, so its float64 autograd gradients
    are the reference for x, weight and bias."""
    t, args = make(case, seed=1)
    s, p, d, G, og, unc = args
    t["offsets"] = np.zeros_like(t["offsets"])
    t["mask"] = None
    g = backward(o, t, args)
    x = torch.tensor(t["x"], dtype=torch.float64, requires_grad=True)
    w = torch.tensor(t["weight"], dtype=torch.float64, requires_grad=True)
    b = torch.tensor(t["bias"], dtype=torch.float64, requires_grad=True)
    pads = tuple(p) if isinstance(p, tuple) else (p, p)
    y = torch.nn.functional.conv1d(torch.nn.functional.pad(x, pads), w, b, stride=s,
                                   dilation=d, groups=G)
    (y * torch.tensor(t["gout"], dtype=torch.float64)).sum().backward()
    for got, ref in ((g["grad_x"], x.grad), (g["grad_weight"], w.grad), (g["grad_bias"], b.grad)):
        assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def all_pins(o):
    for case in CASES:
        pin_finite_differences(o, case)
        pin_conv1d_autograd(o, case)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_backward_matches_finite_differences(case):
    pin_finite_differences(oracle.get(), case)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_backward_matches_conv1d_autograd_for_zero_offsets(case):
    pin_conv1d_autograd(oracle.get(), case)


def test_clamped_taps_pass_no_offset_gradient():
    """Constrained mode, offsets far outside the receptive field: every position is
    clamped, so the offset gradient is exactly zero (and the finite difference agrees)."""
    case = CASES[0]
    t, args = make(case)
    t["offsets"] = np.where(np.arange(t["offsets"].size).reshape(t["offsets"].shape) % 2 == 0,
                            np.float32(50.25), np.float32(-50.25))
    g = backward(oracle.get(), t, args)
    assert np.all(g["grad_offsets"] == 0.0)
    assert np.abs(fd_grad(oracle.get(), t, args, "offsets")).max() == 0.0


BACKWARD_MUTANTS = [
    ("grad_x without the mask", "gx[(b * C_in + ci) * L_in + i0] += m * (1.0 - (double)f) * dv;",
     "gx[(b * C_in + ci) * L_in + i0] += (1.0 - (double)f) * dv;"),
    ("grad_x weights swapped", "gx[(b * C_in + ci) * L_in + i0 + 1] += m * (double)f * dv;",
     "gx[(b * C_in + ci) * L_in + i0 + 1] += m * (1.0 - (double)f) * dv;"),
    ("grad_x drops the left edge", "if (i0 >= 0 && i0 < L_in)", "if (i0 > 0 && i0 < L_in)"),
    ("offset gradient sign", "sum_off += m * (x1 - x0) * dv;", "sum_off += m * (x0 - x1) * dv;"),
    ("offset gradient without mask", "sum_off += m * (x1 - x0) * dv;", "sum_off += (x1 - x0) * dv;"),
    ("clamp gate ignored", "goff[oidx] = sum_off * gate;", "goff[oidx] = sum_off;"),
    ("mask gradient uses x0 only", "sum_mask += ((1.0 - (double)f) * x0 + (double)f * x1) * dv;",
     "sum_mask += x0 * dv;"),
    ("dv with a flipped kernel", "(double)w[(co * cin_g + c) * K + k];",
     "(double)w[(co * cin_g + c) * K + (K - 1 - k)];"),
    ("weight gradient without the mask", "v = v * (double)mask[oidx];", "v = v;"),
    ("bias gradient halved", "acc += (double)gout[(b * C_out + co) * L_out + l];",
     "acc += 0.5 * (double)gout[(b * C_out + co) * L_out + l];"),
    ("dv over all output channels", "for (int64_t co = g * cout_g; co < (g + 1) * cout_g; ++co)\n                            dv",
     "for (int64_t co = 0; co < C_out; ++co)\n                            dv"),
]


@pytest.mark.parametrize("name,old,new", BACKWARD_MUTANTS, ids=[m[0] for m in BACKWARD_MUTANTS])
def test_backward_mutant_is_caught(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = os.path.join(str(tmp_path), "mut.c")
    with open(path, "w") as fh:
        fh.write(src.replace(old, new))
    lib = os.path.join(str(tmp_path), "libmut.so")
    subprocess.run(["gcc", *obuild.CFLAGS, "-w", "-o", lib, path, "-lm"], check=True)
    with pytest.raises(AssertionError):
        all_pins(oracle.Oracle(lib))
