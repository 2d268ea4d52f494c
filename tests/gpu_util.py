"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W

# Normwise bound max|y - r| / max|r| on every output tensor (and every sampled subset).
TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}


_CACHE = {}


def inputs(w, seed):
    """make_inputs with a two-entry cache (the full-size workloads take seconds to draw)."""
    key = (w, seed)
    if key not in _CACHE:
        while len(_CACHE) >= 2:
            _CACHE.pop(next(iter(_CACHE)))
        _CACHE[key] = W.make_inputs(w, seed)
    return _CACHE[key]


def to_dev(t):
    return {k: (v.cuda() if v is not None else None) for k, v in t.items()}


def gpu_forward(w, td, **over):
    a = dict(mask=td["mask"], bias=td["bias"], stride=w.stride, padding=w.padding,
             dilation=w.dilation, groups=w.groups, offset_groups=w.offset_groups,
             unconstrained=w.unconstrained)
    a.update(over)
    return dcn.dcn1d_forward(td["x"], td["offsets"], a["mask"], td["weight"], a["bias"],
                             a["stride"], a["padding"], a["dilation"], a["groups"],
                             a["offset_groups"], a["unconstrained"])


def kernel_name(w, td):
    return dcn.dcn1d_forward_kernel_name(td["x"], td["offsets"], td["mask"], td["weight"],
                                         td["bias"], w.stride, w.padding, w.dilation, w.groups,
                                         w.offset_groups, w.unconstrained)


def oracle_full(w, t):
    return oracle.forward(t["x"], t["offsets"], t["mask"], t["weight"], t["bias"], w.stride,
                          w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)


def oracle_points(w, t, pts):
    return oracle.forward_points(t["x"], t["offsets"], t["mask"], t["weight"], t["bias"],
                                 w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                                 w.unconstrained, pts)


def norm_err(y, r):
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert y.shape == r.shape
    if y.size == 0:
        return 0.0
    assert np.all(np.isfinite(y)), "non-finite GPU output"
    den = np.max(np.abs(r))
    if den == 0.0:
        return float(np.max(np.abs(y)))
    return float(np.max(np.abs(y - r)) / den)


def sample_points(w, n, seed, rows=()):
    """n random (b, co, l) plus every l of the listed (b, co) rows, and the four corners."""
    rng = np.random.default_rng(seed)
    pts = [np.stack([rng.integers(0, w.B, n), rng.integers(0, w.C_out, n),
                     rng.integers(0, w.L_out, n)], axis=1)]
    for b, co in rows:
        L = np.arange(w.L_out)
        pts.append(np.stack([np.full_like(L, b), np.full_like(L, co), L], axis=1))
    corners = [(0, 0, 0), (w.B - 1, w.C_out - 1, w.L_out - 1), (0, w.C_out - 1, 0),
               (w.B - 1, 0, w.L_out - 1)]
    pts.append(np.array(corners))
    return np.concatenate(pts).astype(np.int64)


def reduced(w: W.Workload, **over) -> W.Workload:
    """The same workload with some sizes changed; L_out recomputed by the oracle."""
    import dataclasses
    w2 = dataclasses.replace(w, **over)
    L_out = oracle.out_length(w2.L_in, w2.K, w2.stride, w2.padding, w2.dilation)
    return dataclasses.replace(w2, L_out=L_out, name=w.name + "_reduced")
