"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with an independent source:

* values the pages print (the conv1d examples' lengths and parameter counts,
  the torchvision issue 3673 kh=kw=1 demo output), read from tests/golden/;
* closed forms built from a library routine (torch.nn.functional.conv1d in
  float64 on the CPU), not from the oracle's own formula: zero offsets are the
  conv1d of the "conv1d" page's Description; an integer offset c_k on tap k is
  that tap's conv1d on x shifted by c_k; a fractional offset interpolates
  linearly between the two integer shifts (dc1d page, "Demo notebook");
  constrained-mode saturation equals the conv1d that reads the edge of each
  receptive field;
* invariants: linearity, the bit-exact all-ones mask ("Modulation (DCNv2)"),
  locality of constrained taps;
* hand-worked tiny cases whose arithmetic is written out beside them.

``tests/test_oracle_pins.py`` runs them on the oracle; ``tests/test_oracle_mutants.py``
runs them on deliberately broken copies of the oracle to show each planted
mistake fails at least one pin.
"""
from __future__ import annotations

import fractions
import math
import warnings

import numpy as np
import torch
import torch.nn.functional as F

from conftest import read_golden

# ----------------------------------------------------------------------------- helpers


def conv1d64(x, w, b, s, p, d, groups):
    """torch's conv1d in float64 (library routine, independent of the oracle)."""
    return F.conv1d(x.double(), w.double(), None if b is None else b.double(),
                    stride=s, padding=p, dilation=d, groups=groups)


def tap_shift_conv(x, w, s, p, d, groups, shifts, L_out):
    """Per-tap contributions sum_ci W[co,ci,k] * X(b, ci, l*s - p + k*d + c_k), with X zero
    outside the signal, built from conv1d on a zero-extended, shifted copy of x.

    Returns a float64 tensor [K, B, C_out, L_out] (one slice per tap, bias excluded)."""
    B, C, L = x.shape
    K = w.shape[2]
    cmax = max(abs(int(c)) for c in shifts)
    M = p + cmax + 1
    R = max(0, (L_out - 1) * s - p + (K - 1) * d + cmax - L + 1) + 1
    xe = F.pad(x.double(), (M, R))            # xe[j] = X(j - M)
    outs = []
    for k in range(K):
        wk = torch.zeros_like(w, dtype=torch.float64)
        wk[:, :, k] = w[:, :, k].double()
        start = M - p + int(shifts[k])
        yk = F.conv1d(xe[:, :, start:], wk, None, stride=s, padding=0, dilation=d, groups=groups)
        assert yk.shape[2] >= L_out
        outs.append(yk[:, :, :L_out])
    return torch.stack(outs)


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def rand_case(seed, B, C_in, C_out, K, L_in, s, p, d, groups, og, o, off=None, bias=True,
              mask=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, C_in, L_in, generator=g)
    w = torch.randn(C_out, C_in // groups, K, generator=g)
    b = torch.randn(C_out, generator=g) if bias else None
    L_out = o.out_length(L_in, K, s, p, d)
    assert L_out >= 1
    if off is None:
        offs = torch.zeros(B, og, L_out, K)
    else:
        offs = off(g, (B, og, L_out, K))
    m = torch.rand(B, og, L_out, K, generator=g) if mask else None
    return x, w, b, offs, m, L_out


SHAPES = [
    # B, C_in, C_out, K, L_in, s, p, d, groups, og
    (2, 4, 6, 3, 17, 1, 1, 1, 1, 1),
    (1, 6, 4, 5, 23, 2, 3, 2, 2, 3),
    (3, 8, 8, 4, 19, 3, 0, 1, 4, 2),
    (2, 4, 4, 1, 9, 1, 0, 1, 4, 4),
    (1, 3, 9, 2, 12, 2, 5, 3, 3, 1),
]

# ----------------------------------------------------------------------------- pins


def pin_out_length_page_examples(o):
    """The conv1d page's Examples 1-4: printed output lengths."""
    for row in read_golden("conv1d_shape_examples.txt"):
        _, L_in, _, _, K, s, p, d, _, L_out, _, _ = row
        got = o.out_length(int(L_in), int(K), int(s), int(p), int(d))
        assert got == int(L_out), (row, got)


def pin_out_length_closed_form(o):
    """floor((L_in + 2p - d(K-1) - 1)/s + 1) in exact rational arithmetic; -1 when < 1 or
    when an argument is out of its stated range (K, s, d >= 1, p >= 0)."""
    for L_in in (1, 2, 5, 16, 33):
        for K in (1, 2, 3, 7):
            for s in (1, 2, 3):
                for p in (0, 1, 4):
                    for d in (1, 2, 5):
                        v = math.floor(fractions.Fraction(L_in + 2 * p - d * (K - 1) - 1, s) + 1)
                        want = v if v >= 1 else -1
                        assert o.out_length(L_in, K, s, p, d) == want, (L_in, K, s, p, d)
    for bad in ((0, 3, 1, 0, 1), (8, 0, 1, 0, 1), (8, 3, 0, 0, 1), (8, 3, 1, -1, 1),
                (8, 3, 1, 0, 0)):
        assert o.out_length(*bad) == -1, bad
    # the five named workloads' stated lengths
    for args, want in (((16, 3, 1, 0, 1), 14), ((128, 16, 1, 0, 3), 83),
                       ((16000, 3, 1, 64, 64), 16000), ((4096, 5, 1, 2, 1), 4096),
                       ((8192, 9, 2, 4, 2), 4092)):
        assert o.out_length(*args) == want, args


def pin_weight_shape_page_examples(o):
    """Weight [C_out, C_in/groups, K] plus bias [C_out] reproduces the parameter totals the
    conv1d page prints, and the oracle accepts exactly that weight shape."""
    totals = {}
    for row in read_golden("conv1d_shape_examples.txt"):
        ex, L_in, C_in, C_out, K, s, p, d, groups, L_out, params, extra = row
        C_in, C_out, K, groups = int(C_in), int(C_out), int(K), int(groups)
        key = ex[0]
        n = C_out * (C_in // groups) * K + C_out
        totals[key] = totals.get(key, 0) + n + int(extra)
        if params != "-":
            assert totals[key] == int(params), (ex, totals[key], params)
        x = torch.randn(1, C_in, int(L_in))
        w = torch.randn(C_out, C_in // groups, K)
        offs = torch.zeros(1, 1, int(L_out), K)
        y = o.forward(x, offs, None, w, torch.zeros(C_out), int(s), int(p), int(d), groups, 1,
                      False)
        assert y.shape == (1, C_out, int(L_out))
        assert rel_err(y, conv1d64(x, w, None, int(s), int(p), int(d), groups)) < 1e-12


def pin_zero_offsets_equal_conv1d(o):
    """Zero offsets reproduce the conv1d Description exactly (dc1d "Going faster": the
    zero-offset invariant); constrained mode changes nothing at zero offsets."""
    for i, (B, Ci, Co, K, L, s, p, d, G, og) in enumerate(SHAPES):
        x, w, b, offs, _, L_out = rand_case(100 + i, B, Ci, Co, K, L, s, p, d, G, og, o)
        ref = conv1d64(x, w, b, s, p, d, G)
        for unc in (False, True):
            y = o.forward(x, offs, None, w, b, s, p, d, G, og, unc)
            assert y.shape == tuple(ref.shape)
            assert rel_err(y, ref) < 1e-12, (i, unc)


def pin_integer_offsets_are_shifts(o):
    """A constant integer offset c_k on tap k reads x shifted by c_k (dc1d "Demo notebook":
    an integer offset is an exact shift), with zero fill past both ends."""
    for i, (B, Ci, Co, K, L, s, p, d, G, og) in enumerate(SHAPES):
        x, w, b, _, _, L_out = rand_case(200 + i, B, Ci, Co, K, L, s, p, d, G, og, o)
        rng = np.random.default_rng(i)
        shifts = rng.integers(-4, 5, size=K)
        shifts[0] = -(L + 3)                   # one tap entirely outside the signal
        offs = torch.tensor(shifts, dtype=torch.float32).expand(B, og, L_out, K).contiguous()
        ref = tap_shift_conv(x, w, s, p, d, G, shifts, L_out).sum(0)
        if b is not None:
            ref = ref + b.double()[None, :, None]
        y = o.forward(x, offs, None, w, b, s, p, d, G, og, True)
        assert rel_err(y, ref) < 1e-12, (i, shifts)


def pin_fractional_offsets_interpolate(o):
    """A fractional offset c + f mixes the shifts c and c+1 with weights (1-f) and f (dc1d
    "Demo notebook"; the 1D case of the bilinear weights in the deformable-convolution
    article, "Step 2")."""
    for i, (B, Ci, Co, K, L, s, p, d, G, og) in enumerate(SHAPES):
        x, w, b, _, _, L_out = rand_case(300 + i, B, Ci, Co, K, L, s, p, d, G, og, o)
        rng = np.random.default_rng(50 + i)
        c = rng.integers(-3, 4, size=K)
        f = rng.choice([0.125, 0.25, 0.5, 0.75, 0.875], size=K)
        offs = torch.tensor(c + f, dtype=torch.float32).expand(B, og, L_out, K).contiguous()
        lo = tap_shift_conv(x, w, s, p, d, G, c, L_out)
        hi = tap_shift_conv(x, w, s, p, d, G, c + 1, L_out)
        fk = torch.tensor(f, dtype=torch.float64)[:, None, None, None]
        ref = ((1 - fk) * lo + fk * hi).sum(0)
        y = o.forward(x, offs, None, w, None, s, p, d, G, og, True)
        assert rel_err(y, ref) < 1e-12, (i, c, f)


def pin_worked_example_torchvision_issue(o):
    """torchvision issue 3673 kh=kw=1 demo, restated in 1D along each axis."""
    rows = read_golden("torchvision_issue3673_kh1kw1.txt")
    printed = {}
    for co, h, *vals in rows:
        printed[(int(co[2:]), int(h[1:]))] = [float(v) for v in vals]
    x2 = torch.arange(27, dtype=torch.float32).reshape(3, 3, 3)         # x[c, h, w]
    W = torch.tensor([[1, 0, 0], [0, 1, 0], [1, 1, 0], [0, 0, 1], [0, 1, 0]], dtype=torch.float32)
    # Width direction: signals along w, one per row h (batch = h); channels 0, 1 with
    # offset groups 0 (dx = -1) and 1 (dx = +1).  Out channels 0, 1, 2, 4 read only them.
    xw = x2[:2].permute(1, 0, 2).contiguous()                          # [h, c, w]
    offs = torch.tensor([-1.0, 1.0]).reshape(1, 2, 1, 1).expand(3, 2, 3, 1).contiguous()
    sel = [0, 1, 2, 4]
    wsel = W[sel][:, :2].reshape(4, 2, 1).contiguous()
    y = o.forward(xw, offs, None, wsel, None, 1, 0, 1, 1, 2, True)     # [h, co, w]
    for j, co in enumerate(sel):
        for h in range(3):
            assert list(y[h, j]) == printed[(co, h)], (co, h, y[h, j])
    # Height direction: signals along h, one per column w (batch = w); channel 2, dy = -1.
    xh = x2[2].t().contiguous().reshape(3, 1, 3)                        # [w, 1, h]
    offs = torch.full((3, 1, 3, 1), -1.0)
    y = o.forward(xh, offs, None, torch.ones(1, 1, 1), None, 1, 0, 1, 1, 1, True)
    for h in range(3):
        assert [y[w_, 0, h] for w_ in range(3)] == printed[(3, h)], (h, y[:, 0, h])


def pin_hand_cases(o):
    """Tiny cases worked by hand from the definition (values are dyadic, so exact)."""
    x = torch.tensor([[[1.0, 2.0, 4.0, 8.0, 16.0, 32.0]]])
    one = torch.ones(1, 1, 1)

    # K=1, offset +0.5 everywhere: (x[l] + x[l+1]) / 2, and x[6] reads 0.
    offs = torch.full((1, 1, 6, 1), 0.5)
    y = o.forward(x, offs, None, one, None, 1, 0, 1, 1, 1, True)
    assert list(y[0, 0]) == [1.5, 3.0, 6.0, 12.0, 24.0, 16.0]

    # K=1, offset -0.25: pos = l - 0.25, i0 = l-1, f = 0.75: 0.25 x[l-1] + 0.75 x[l].
    offs = torch.full((1, 1, 6, 1), -0.25)
    y = o.forward(x, offs, None, one, None, 1, 0, 1, 1, 1, True)
    assert list(y[0, 0]) == [0.75, 1.75, 3.5, 7.0, 14.0, 28.0]

    # K=2, d=2, p=1, constrained, W = [1, 10].  Receptive field of l: [l-1, l+1].
    # tap 0: base l-1, offset +0.5 -> pos l-0.5 (inside): 0.5 (X(l-1) + X(l)).
    # tap 1: base l+1, offset -3 -> pos l-2, clamped to l-1: X(l-1).
    w = torch.tensor([[[1.0, 10.0]]])
    offs = torch.tensor([0.5, -3.0]).expand(1, 1, 6, 2).contiguous()
    y = o.forward(x, offs, None, w, None, 1, 1, 2, 1, 1, False)
    assert list(y[0, 0]) == [0.5, 11.5, 23.0, 46.0, 92.0, 184.0]
    # Same, unconstrained: tap 1 reads X(l-2) instead.
    y = o.forward(x, offs, None, w, None, 1, 1, 2, 1, 1, True)
    assert list(y[0, 0]) == [0.5, 1.5, 13.0, 26.0, 52.0, 104.0]

    # Mask scales each sampled value (K=1, zero offset): [1*0.5, 2*2, 4*0, 8*1].
    x4 = torch.tensor([[[1.0, 2.0, 4.0, 8.0]]])
    m = torch.tensor([0.5, 2.0, 0.0, 1.0]).reshape(1, 1, 4, 1)
    y = o.forward(x4, torch.zeros(1, 1, 4, 1), m, one, None, 1, 0, 1, 1, 1, False)
    assert list(y[0, 0]) == [0.5, 4.0, 0.0, 8.0]

    # Conv groups: two independent channels, weights 3 and 5, bias 1 and -1.
    xg = torch.tensor([[[1.0, 2.0], [10.0, 20.0]]])
    wg = torch.tensor([3.0, 5.0]).reshape(2, 1, 1)
    y = o.forward(xg, torch.zeros(1, 1, 2, 1), None, wg, torch.tensor([1.0, -1.0]), 1, 0, 1, 2,
                  1, False)
    assert y[0].tolist() == [[4.0, 7.0], [49.0, 99.0]]

    # Offset groups: channel 0 moves by +1, channel 1 by -1; out = sum of both.
    xo = torch.tensor([[[1.0, 2.0, 4.0], [10.0, 20.0, 40.0]]])
    offs = torch.tensor([1.0, -1.0]).reshape(1, 2, 1, 1).expand(1, 2, 3, 1).contiguous()
    y = o.forward(xo, offs, None, torch.ones(1, 2, 1), None, 1, 0, 1, 1, 2, True)
    assert list(y[0, 0]) == [2.0 + 0.0, 4.0 + 10.0, 0.0 + 20.0]

    # Stride 2, padding 1, K=3, integer offsets: l in {0,1,2}; taps at 2l-1, 2l, 2l+1.
    # Offsets (+1, 0, -2) unconstrained: reads X(2l), X(2l), X(2l-1) with W = (1, 2, 4).
    w3 = torch.tensor([[[1.0, 2.0, 4.0]]])
    offs = torch.tensor([1.0, 0.0, -2.0]).expand(1, 1, 3, 3).contiguous()
    y = o.forward(x, offs, None, w3, None, 2, 1, 1, 1, 1, True)
    # l=0: X0 + 2 X0 + 4 X(-1) = 1 + 2 + 0 = 3
    # l=1: X2 + 2 X2 + 4 X1 = 4 + 8 + 8 = 20
    # l=2: X4 + 2 X4 + 4 X3 = 16 + 32 + 32 = 80
    assert list(y[0, 0]) == [3.0, 20.0, 80.0]


def pin_linearity(o):
    """Linear in x, in the weight and in the mask; the bias adds."""
    B, Ci, Co, K, L, s, p, d, G, og = SHAPES[1]
    normal = lambda g, sh: torch.randn(sh, generator=g) * 2.5
    x1, w1, b, offs, m1, _ = rand_case(400, B, Ci, Co, K, L, s, p, d, G, og, o, off=normal,
                                       mask=True)
    x2, w2, _, _, m2, _ = rand_case(401, B, Ci, Co, K, L, s, p, d, G, og, o, mask=True)
    # Round the operands to 8 significant bits so the dyadic combinations below are exact
    # in float32 (the oracle's input type); only the oracle's own rounding remains.
    q = lambda t: t.to(torch.bfloat16).float()
    x1, w1, m1, x2, w2, m2 = (q(t) for t in (x1, w1, m1, x2, w2, m2))
    for unc in (False, True):
        f = lambda x, w, m, bb: o.forward(x, offs, m, w, bb, s, p, d, G, og, unc)
        base = f(x1, w1, m1, None)
        assert rel_err(f(1.5 * x1 - 0.25 * x2, w1, m1, None),
                       1.5 * base - 0.25 * f(x2, w1, m1, None)) < 1e-12
        assert rel_err(f(x1, 0.5 * w1 + 2.0 * w2, m1, None),
                       0.5 * base + 2.0 * f(x1, w2, m1, None)) < 1e-12
        assert rel_err(f(x1, w1, 0.75 * m1 + 0.5 * m2, None),
                       0.75 * base + 0.5 * f(x1, w1, m2, None)) < 1e-12
        assert rel_err(f(x1, w1, m1, b), base + b.double().numpy()[None, :, None]) < 1e-12


def pin_mask_ones_bitwise(o):
    """dc1d "Modulation (DCNv2)": an all-ones mask is bit-for-bit the same as no mask."""
    for i, (B, Ci, Co, K, L, s, p, d, G, og) in enumerate(SHAPES):
        normal = lambda g, sh: torch.randn(sh, generator=g) * 3.0
        x, w, b, offs, _, L_out = rand_case(500 + i, B, Ci, Co, K, L, s, p, d, G, og, o,
                                            off=normal)
        for unc in (False, True):
            a = o.forward(x, offs, None, w, b, s, p, d, G, og, unc)
            c = o.forward(x, offs, torch.ones_like(offs), w, b, s, p, d, G, og, unc)
            assert np.array_equal(a.view(np.int64), c.view(np.int64))


def pin_constrained_saturation(o):
    """Constrained mode, reading of "each kernel tap is constrained to its own receptive
    field": huge positive offsets read the right edge l*s-p+d(K-1) of the field, huge
    negative ones its left edge l*s-p, for every tap (a conv1d with shifted taps)."""
    for i, (B, Ci, Co, K, L, s, p, d, G, og) in enumerate(SHAPES):
        x, w, b, _, _, L_out = rand_case(600 + i, B, Ci, Co, K, L, s, p, d, G, og, o)
        for sign, shifts in ((1.0, [d * (K - 1 - k) for k in range(K)]),
                             (-1.0, [-k * d for k in range(K)])):
            offs = torch.full((B, og, L_out, K), sign * 1.0e4)
            ref = tap_shift_conv(x, w, s, p, d, G, shifts, L_out).sum(0) + b.double()[None, :, None]
            y = o.forward(x, offs, None, w, b, s, p, d, G, og, False)
            assert rel_err(y, ref) < 1e-12, (i, sign)


def pin_constrained_locality(o):
    """Constrained taps only read inside [l*s-p, l*s-p+d(K-1)+1]: changing x anywhere else
    leaves out[:, :, l] bit-for-bit unchanged."""
    B, Ci, Co, K, L, s, p, d, G, og = SHAPES[1]
    big = lambda g, sh: torch.randn(sh, generator=g) * 20.0
    x, w, b, offs, _, L_out = rand_case(700, B, Ci, Co, K, L, s, p, d, G, og, o, off=big)
    y = o.forward(x, offs, None, w, b, s, p, d, G, og, False)
    for l in range(L_out):
        lo, hi = l * s - p, l * s - p + d * (K - 1) + 1
        x2 = x.clone()
        keep = torch.zeros(L, dtype=torch.bool)
        keep[max(lo, 0):max(min(hi + 1, L), 0)] = True
        x2[:, :, ~keep] = torch.randn(x2[:, :, ~keep].shape) * 100.0
        y2 = o.forward(x2, offs, None, w, b, s, p, d, G, og, False)
        assert np.array_equal(y[:, :, l], y2[:, :, l]), l


def pin_sample_index(o):
    """Floor/fraction of the sampling position: i0 + f reproduces the float32 position,
    0 <= f < 1, and the constrained position stays in the receptive field."""
    g = torch.Generator().manual_seed(800)
    B, G, L_in, K, s, p, d = 2, 3, 40, 4, 2, 5, 3
    L_out = o.out_length(L_in, K, s, p, d)
    offs = torch.randn(B, G, L_out, K, generator=g) * 7.0
    offs[0, 0, :, 0] = torch.tensor([-2.5, -1.0, -0.0, 0.0, 1.0, 2.5] * 10)[:L_out]
    for unc in (False, True):
        i0, fr = o.sample_index(offs, L_in, K, s, p, d, unc)
        assert i0.dtype == np.int32 and fr.dtype == np.float32
        assert np.all(fr >= 0.0) and np.all(fr < 1.0)
        l = np.arange(L_out)[None, None, :, None]
        k = np.arange(K)[None, None, None, :]
        base = (l * s - p + k * d).astype(np.float32)
        pos = base + offs.numpy()                       # float32 + float32, round to nearest
        if not unc:
            pos = np.minimum(np.maximum(pos, (l * s - p).astype(np.float32)),
                             (l * s - p + d * (K - 1)).astype(np.float32))
        assert np.array_equal(i0.astype(np.float32) + fr, pos)
        assert np.array_equal(i0, np.floor(pos).astype(np.int32))
    # bf16 offsets widen exactly: the same values give the same taps.
    ob = offs.to(torch.bfloat16)
    a = o.sample_index(ob, L_in, K, s, p, d, True)
    c = o.sample_index(ob.float(), L_in, K, s, p, d, True)
    assert np.array_equal(a[0], c[0]) and np.array_equal(a[1], c[1])


def pin_offset_group_reading(o):
    """READING, not a page value: channel ci uses offset group ci // (C_in / offset_groups)
    (contiguous blocks, the torchvision convention; the dc1d page only says offset_groups
    divides C_in).  Checked as: offset_groups = G with offsets O equals offset_groups = C_in
    with each group's offsets repeated over its block of channels.  The pages do not fix
    this mapping, so it is parity unpinned against them."""
    B, Ci, Co, K, L, s, p, d, G, og = 2, 6, 4, 3, 15, 1, 2, 2, 1, 3
    normal = lambda g, sh: torch.randn(sh, generator=g) * 2.0
    x, w, b, offs, m, L_out = rand_case(900, B, Ci, Co, K, L, s, p, d, G, og, o, off=normal,
                                        mask=True)
    rep = Ci // og
    offs_c = offs.repeat_interleave(rep, dim=1).contiguous()
    m_c = m.repeat_interleave(rep, dim=1).contiguous()
    for unc in (False, True):
        a = o.forward(x, offs, m, w, b, s, p, d, G, og, unc)
        c = o.forward(x, offs_c, m_c, w, b, s, p, d, G, Ci, unc)
        assert np.array_equal(a, c)


def pin_asymmetric_padding(o):
    """Padding given per side: zero offsets equal torch's conv1d on the explicitly padded
    signal (F.pad, library routine) with padding 0; the dc1d page's "same" (stride 1,
    d(K-1) odd: d(K-1)//2 on the left, the rest on the right) equals torch's own
    padding="same" and keeps L_out = L_in."""
    cases = [  # B, C_in, C_out, K, L_in, s, (pl, pr), d, groups, og
        (2, 4, 6, 4, 15, 1, (1, 2), 1, 2, 2),
        (1, 6, 3, 3, 20, 2, (0, 3), 2, 3, 1),
        (2, 4, 4, 2, 11, 1, (2, 0), 3, 4, 4),
    ]
    for i, (B, Ci, Co, K, L, s, pads, d, G, og) in enumerate(cases):
        g = torch.Generator().manual_seed(700 + i)
        x = torch.randn(B, Ci, L, generator=g)
        w = torch.randn(Co, Ci // G, K, generator=g)
        b = torch.randn(Co, generator=g)
        L_out = o.out_length(L, K, s, pads, d)
        ref = F.conv1d(F.pad(x.double(), pads), w.double(), b.double(), stride=s, dilation=d,
                       groups=G)
        assert L_out == ref.shape[2], (i, L_out, ref.shape)
        offs = torch.zeros(B, og, L_out, K)
        for unc in (False, True):
            y = o.forward(x, offs, None, w, b, s, pads, d, G, og, unc)
            assert rel_err(y, ref) < 1e-12, (i, unc)
    for K, d in ((4, 1), (2, 3), (6, 1)):   # d(K-1) odd: one more zero on the right
        g = torch.Generator().manual_seed(800 + K)
        x = torch.randn(2, 3, 16, generator=g)
        w = torch.randn(5, 3, K, generator=g)
        tot = d * (K - 1)
        pads = (tot // 2, tot - tot // 2)
        assert o.out_length(16, K, 1, pads, d) == 16
        with warnings.catch_warnings():   # torch notes that it pads a copy for this case
            warnings.simplefilter("ignore", UserWarning)
            ref = F.conv1d(x.double(), w.double(), None, padding="same", dilation=d)
        y = o.forward(x, torch.zeros(2, 1, 16, K), None, w, None, 1, pads, d, 1, 1, False)
        assert rel_err(y, ref) < 1e-12, (K, d)


ALL_PINS = [
    pin_out_length_page_examples,
    pin_out_length_closed_form,
    pin_weight_shape_page_examples,
    pin_zero_offsets_equal_conv1d,
    pin_integer_offsets_are_shifts,
    pin_fractional_offsets_interpolate,
    pin_worked_example_torchvision_issue,
    pin_hand_cases,
    pin_linearity,
    pin_mask_ones_bitwise,
    pin_constrained_saturation,
    pin_constrained_locality,
    pin_sample_index,
    pin_offset_group_reading,
    pin_asymmetric_padding,
]
