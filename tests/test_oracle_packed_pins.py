"""Pins of the oracle's PackedDeformConv1d trunk and layer (test infrastructure, CPU only).

The trunk ("dc1d (DeformConv1d)" page, "PackedDeformConv1d" and "Modulation (DCNv2)") is a
depthwise convolution followed by pointwise projections to the offsets and, when modulated,
through a sigmoid to the mask.  It is pinned by:

- torch's float64 conv1d (groups = C_in, then 1x1 convolutions) and torch.sigmoid, a
  library routine the oracle does not use, on random cases that cover strides, dilation,
  per-side padding, absent biases and several offset groups;
- a worked example computed by hand (below), which fixes the channel order g*K + k;
- the page's statement on the zero-initialised mask projection: every tap's mask is exactly
  0.5, so the modulated layer's output minus its bias is half the unmodulated one.
Planted mistakes in copies of the trunk must each fail one of these pins.
"""
import os
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import build as obuild

# B, C_in, C_out, K, L_in, stride, padding, dilation, groups, offset_groups, modulated, biases
CASES = [
    (2, 8, 8, 3, 40, 1, (4, 4), 4, 8, 8, True, True),     # the page's example, scaled down
    (1, 6, 4, 4, 23, 2, (1, 2), 1, 2, 3, True, True),
    (2, 4, 6, 2, 17, 1, 0, 3, 1, 2, False, True),
    (1, 8, 8, 5, 30, 1, (2, 2), 2, 1, 4, True, False),
]
IDS = ["page_example_same", "strided_asymmetric_og3", "valid_dil3_unmodulated",
       "no_biases_og4"]


def make(case, seed=0):
    B, Ci, Co, K, L, s, p, d, G, og, modulated, biases = case
    g = torch.Generator().manual_seed(seed)
    r = lambda *shape: torch.randn(*shape, generator=g, dtype=torch.float64)  # noqa: E731
    t = {
        "x": r(B, Ci, L).float(),
        "dw_weight": r(Ci, 1, K).float(),
        "dw_bias": r(Ci).float() if biases else None,
        "off_weight": (0.5 * r(og * K, Ci)).float(),
        "off_bias": r(og * K).float() if biases else None,
        "mask_weight": (0.5 * r(og * K, Ci)).float() if modulated else None,
        "mask_bias": r(og * K).float() if (modulated and biases) else None,
        "weight": r(Co, Ci // G, K).float(),
        "bias": r(Co).float() if biases else None,
    }
    return t, dict(stride=s, padding=p, dilation=d, groups=G, offset_groups=og, K=K)


def trunk(o, t, a):
    return o.packed_trunk(t["x"], t["dw_weight"], t["dw_bias"], t["off_weight"], t["off_bias"],
                          t["mask_weight"], t["mask_bias"], a["K"], a["stride"], a["padding"],
                          a["dilation"], a["offset_groups"])


def torch_trunk(t, a):
    """The same block from torch's float64 conv1d and sigmoid."""
    x = t["x"].double()
    pads = a["padding"] if isinstance(a["padding"], tuple) else (a["padding"],) * 2
    C = x.shape[1]
    og, K = a["offset_groups"], a["K"]
    dwb = t["dw_bias"].double() if t["dw_bias"] is not None else None
    mid = F.conv1d(F.pad(x, pads), t["dw_weight"].double(), dwb, stride=a["stride"],
                   dilation=a["dilation"], groups=C)

    def project(w, b):
        z = F.conv1d(mid, w.double()[:, :, None], b.double() if b is not None else None)
        B, _, L_out = z.shape
        return z.view(B, og, K, L_out).permute(0, 1, 3, 2).numpy()

    off = project(t["off_weight"], t["off_bias"])
    mask = None
    if t["mask_weight"] is not None:
        mask = torch.sigmoid(torch.from_numpy(project(t["mask_weight"], t["mask_bias"]))).numpy()
    return off, mask


def pin_torch_composition(o, case):
    t, a = make(case)
    off, mask = trunk(o, t, a)
    roff, rmask = torch_trunk(t, a)
    assert off.shape == roff.shape
    assert np.allclose(off, roff, rtol=1e-12, atol=1e-12)
    assert (mask is None) == (rmask is None)
    if mask is not None:
        assert np.allclose(mask, rmask, rtol=1e-12, atol=1e-12)


# Worked example by hand: x = [1, 2, 3, 4], K = 2, stride 1, no padding, dilation 1, one
# offset group.  Depthwise weight (0.5, -1), bias 0.25:
#   t = 0.25 + 0.5 x[l] - x[l+1] = (-1.25, -1.75, -2.25) for l = 0, 1, 2.
# Offset projection (channel j = g*K + k): weights (2, -1), biases (0.5, 0):
#   offsets[l] = (0.5 + 2 t, -t) = (-2, 1.25), (-3, 1.75), (-4, 2.25).
# Mask projection: weights (1, 0), biases (0, 0): mask[l] = (sigmoid(t), 0.5), where
#   sigmoid(-1.25) = 0.22270013882530884, sigmoid(-1.75) = 0.14804719803168948,
#   sigmoid(-2.25) = 0.09534946489910949.
WORKED_OFFSETS = [[-2.0, 1.25], [-3.0, 1.75], [-4.0, 2.25]]
WORKED_MASK = [[0.22270013882530884, 0.5], [0.14804719803168948, 0.5],
               [0.09534946489910949, 0.5]]


def pin_worked_example(o):
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]], np.float32)
    off, mask = o.packed_trunk(x, np.array([[[0.5, -1.0]]], np.float32),
                               np.array([0.25], np.float32), np.array([[2.0], [-1.0]], np.float32),
                               np.array([0.5, 0.0], np.float32),
                               np.array([[1.0], [0.0]], np.float32),
                               np.array([0.0, 0.0], np.float32), 2, 1, 0, 1, 1)
    assert off.shape == (1, 1, 3, 2)
    assert np.array_equal(off[0, 0], np.array(WORKED_OFFSETS))
    assert np.allclose(mask[0, 0], np.array(WORKED_MASK), rtol=1e-13, atol=0)


def pin_zero_initialised_mask_halves_the_output(o, case):
    t, a = make(case, seed=3)
    if t["mask_weight"] is None:
        t["mask_weight"] = torch.zeros(a["offset_groups"] * a["K"], t["x"].shape[1])
    t["mask_weight"] = torch.zeros_like(t["mask_weight"])
    t["mask_bias"] = torch.zeros(a["offset_groups"] * a["K"])
    args = (a["stride"], a["padding"], a["dilation"], a["groups"], a["offset_groups"], False)
    y_mod, _, mask = o.packed_forward(t["x"], t["dw_weight"], t["dw_bias"], t["off_weight"],
                                      t["off_bias"], t["mask_weight"], t["mask_bias"],
                                      t["weight"], t["bias"], *args)
    y_plain, _, none = o.packed_forward(t["x"], t["dw_weight"], t["dw_bias"], t["off_weight"],
                                        t["off_bias"], None, None, t["weight"], t["bias"], *args)
    assert none is None and np.all(mask == 0.5)
    b = t["bias"].double().numpy()[None, :, None] if t["bias"] is not None else 0.0
    assert np.allclose(y_mod - b, 0.5 * (y_plain - b), rtol=1e-12, atol=1e-12)
    assert np.abs(y_plain - b).max() > 0.1


def all_pins(o):
    pin_worked_example(o)
    for case in CASES:
        pin_torch_composition(o, case)
        pin_zero_initialised_mask_halves_the_output(o, case)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_trunk_matches_torch_conv1d_composition(case):
    pin_torch_composition(oracle.get(), case)


def test_trunk_worked_example():
    pin_worked_example(oracle.get())


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_zero_initialised_mask_halves_the_output(case):
    pin_zero_initialised_mask_halves_the_output(oracle.get(), case)


def test_trunk_rejects_bad_shapes():
    t, a = make(CASES[1])
    with pytest.raises(ValueError):
        oracle.packed_trunk(t["x"], t["dw_weight"], None, t["off_weight"], None, None, None,
                            a["K"], a["stride"], a["padding"], a["dilation"], 4)


TRUNK_MUTANTS = [
    ("depthwise bias dropped", "double acc = dw_b ? (double)dw_b[c] : 0.0;", "double acc = 0.0;"),
    ("depthwise taps flipped", "acc += (double)dw_w[c * K + k] * xv;",
     "acc += (double)dw_w[c * K + (K - 1 - k)] * xv;"),
    ("trunk ignores the left padding", "int64_t i = l * stride - padding + k * dilation;",
     "int64_t i = l * stride + k * dilation;"),
    ("trunk without dilation", "int64_t i = l * stride - padding + k * dilation;",
     "int64_t i = l * stride - padding + k;"),
    ("tap-major channel order", "int64_t g = j / K, k = j % K;",
     "int64_t g = j % offset_groups, k = j / offset_groups;"),
    ("offset bias dropped", "double z = off_b ? (double)off_b[j] : 0.0;", "double z = 0.0;"),
    ("pointwise weight transposed", "z += (double)off_w[j * C_in + c] * t[c];",
     "z += (double)off_w[c * J + j] * t[c];"),
    ("mask branch reuses the offset weights", "zm += (double)mask_w[j * C_in + c] * t[c];",
     "zm += (double)off_w[j * C_in + c] * t[c];"),
    ("sigmoid missing", "mask_out[oidx] = 1.0 / (1.0 + exp(-zm));", "mask_out[oidx] = zm;"),
]


@pytest.mark.parametrize("name,old,new", TRUNK_MUTANTS, ids=[m[0] for m in TRUNK_MUTANTS])
def test_trunk_mutant_is_caught(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = os.path.join(str(tmp_path), "mut.c")
    with open(path, "w") as fh:
        fh.write(src.replace(old, new))
    lib = os.path.join(str(tmp_path), "libmut.so")
    subprocess.run(["gcc", *obuild.CFLAGS, "-w", "-o", lib, path, "-lm"], check=True)
    with pytest.raises(AssertionError):
        all_pins(oracle.Oracle(lib))
