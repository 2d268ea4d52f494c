"""The CPU oracle against the pages and the mathematics (no GPU)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.get())


def test_forward_points_matches_forward():
    """The per-point entry computes the same numbers as the full one."""
    import numpy as np
    import torch
    import workloads as W

    w, t = W.small_case(3, B=2, C_in=6, C_out=4, K=3, stride=2, padding=2, dilation=2,
                        groups=2, offset_groups=3, L_in=21, L_out=oracle.out_length(21, 3, 2, 2, 2),
                        mask=True, unconstrained=False)
    args = (t["x"], t["offsets"], t["mask"], t["weight"], t["bias"], w.stride, w.padding,
            w.dilation, w.groups, w.offset_groups, w.unconstrained)
    full = oracle.forward(*args)
    pts = np.array([(b, co, l) for b in range(2) for co in range(4) for l in range(w.L_out)])
    got = oracle.forward_points(*args, pts)
    assert np.array_equal(got, full.reshape(-1))


def test_named_workload_tiny_runs():
    import workloads as W
    w = W.TINY_F32
    t = W.make_inputs(w)
    y = oracle.forward(t["x"], t["offsets"], t["mask"], t["weight"], t["bias"], w.stride,
                       w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    assert y.shape == (1, 4, 14)
