"""Inputs that expose the integer side of the sampling step in the OUTPUT of every kernel.

The forward is continuous in the offsets, so an output compared within a tolerance cannot
show a wrong floor, clamp or neighbour choice on a single tap among thousands.  These
inputs make every such choice visible bit for bit:

* x holds small non-zero integers (magnitude 1..8) and neighbouring positions always
  differ, so reading a wrong neighbour changes a sampled value by at least 1/4;
* every offset is a multiple of 1/4, so each fraction f is 0, 1/4, 1/2 or 3/4 and the
  interpolation ``x0 + f (x1 - x0)`` is exact in bf16, fp16 and fp32;
* the weights are one-hot (each output channel reads exactly one (channel, tap) column of
  the reduction; calls with shifted weights cover every column), and the mask takes the
  values 1/4, 1/2, 1 and 2, so each output is one sampled value scaled exactly;
* the offsets mix integers and quarters near the receptive field, values that land
  exactly on the constrained clamp bounds or a quarter beyond them, values that cross the
  32-position margin the fast kernels stage around their windows, and values far past
  both ends of the signal.

With these inputs each output of a kernel equals the oracle's exact result rounded to the
dtype, so the tests compare with ``torch.equal``.  ``near_integer`` adds offsets a few ulp
either side of an integer; their interpolation is exact only in fp32 (a single rounding of
a value that needs more than 16 bits), so only fp32 kernels take them.

This module draws inputs only; it holds none of the method's arithmetic.
"""
from __future__ import annotations

import torch


def probe_x(shape, gen: torch.Generator) -> torch.Tensor:
    """Signed integers of magnitude 1..8 along the last axis, neighbours always distinct."""
    steps = torch.randint(1, 8, shape, generator=gen)            # 1..7: never 0 mod 8
    mag = 1 + torch.remainder(torch.cumsum(steps, dim=-1), 8)    # 1..8, changes every step
    sign = torch.randint(0, 2, shape, generator=gen) * 2 - 1
    return (mag * sign).float()


def probe_offsets(shape, K: int, dilation: int, gen: torch.Generator,
                  near_integer: bool = False) -> torch.Tensor:
    """[B, G, L_out, K] offsets from the mixture the module docstring describes."""
    n = 1
    for s in shape:
        n *= s
    k = torch.arange(n) % K                       # the tap of each element (K is innermost)
    kind = torch.randint(0, 10, (n,), generator=gen)
    quarter = torch.randint(0, 4, (n,), generator=gen).float() * 0.25
    sign = (torch.randint(0, 2, (n,), generator=gen) * 2 - 1).float()
    small = torch.randint(-4, 5, (n,), generator=gen).float()
    mid = torch.randint(20, 45, (n,), generator=gen).float() * sign
    far = torch.randint(100, 3000, (n,), generator=gen).float() * sign
    lo_hit = -(k * dilation).float()              # constrained: the position lands on lo
    hi_hit = ((K - 1 - k) * dilation).float()     # ... and on hi
    off = small + quarter                         # kinds 0-3
    off = torch.where(kind == 4, small, off)
    off = torch.where(kind == 5, lo_hit - torch.where(quarter > 0.3, quarter, 0.0), off)
    off = torch.where(kind == 6, hi_hit + torch.where(quarter > 0.3, quarter, 0.0), off)
    off = torch.where(kind == 7, mid + quarter, off)
    off = torch.where(kind == 8, far + quarter, off)
    if near_integer:
        e = torch.randint(8, 24, (n,), generator=gen).float()
        off = torch.where(kind == 9, small + sign * torch.pow(2.0, -e), off)
    else:
        off = torch.where(kind == 9, small + 0.5, off)
    return off.reshape(shape)


def probe_mask(shape, gen: torch.Generator) -> torch.Tensor:
    """Mask values 1/4, 1/2, 1 and 2 (scaling by them is exact)."""
    return torch.pow(2.0, torch.randint(-2, 2, shape, generator=gen).float())


def onehot_weight(C_out: int, C_in: int, K: int, groups: int, shift: int) -> torch.Tensor:
    """[C_out, C_in/groups, K]: output channel co of each conv group reads reduction column
    (co_local + shift) mod (C_in/groups * K), with the column index c*K + k."""
    cin_g, cout_g = C_in // groups, C_out // groups
    ncols = cin_g * K
    w = torch.zeros(C_out, cin_g * K)
    co = torch.arange(C_out)
    w[co, (co % cout_g + shift) % ncols] = 1.0
    return w.reshape(C_out, cin_g, K)


def shifts_covering(C_out: int, C_in: int, K: int, groups: int):
    """Weight shifts whose one-hot weights together read every reduction column."""
    ncols = (C_in // groups) * K
    cout_g = C_out // groups
    return list(range(0, ncols, cout_g))


def probe_inputs(B, C_in, L_in, L_out, K, dilation, offset_groups, mask, seed,
                 near_integer=False) -> dict:
    """x, offsets and (optionally) mask of a probe case, float32 on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    x = probe_x((B, C_in, L_in), gen)
    off = probe_offsets((B, offset_groups, L_out, K), K, dilation, gen, near_integer)
    m = probe_mask(off.shape, gen) if mask else None
    return {"x": x, "offsets": off, "mask": m}
