"""CPU oracle for the 1D deformable convolution forward and backward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it never imports the product path.

The arithmetic lives in ``dcn1d_oracle.c`` (plain loops, double accumulation,
float32 sampling positions); this module only marshals arrays.  bf16 inputs are
widened to float32 exactly before they reach the C code.

Parity status: every function is pinned by ``tests/test_oracle_pins.py`` (forward)
and ``tests/test_oracle_backward_pins.py`` (backward: finite differences of the
forward, conv1d autograd for zero offsets) and ``tests/test_oracle_packed_pins.py``
(PackedDeformConv1d's offset and mask trunk: torch's float64 conv1d composition, a worked
example by hand, the zero-initialised mask halving the output) except the exact clamp bounds of
constrained mode, which no page fixes; those are checked only through invariants
(locality, saturation) and are "parity unpinned" as to the bounds themselves.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np
import torch

from . import build as _build

_i64 = ctypes.c_int64
_int = ctypes.c_int
_p = ctypes.c_void_p


def _f32(t):
    """float32 contiguous numpy copy (bf16 -> f32 widening is exact)."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return np.ascontiguousarray(t.detach().cpu().to(torch.float32).numpy())
    return np.ascontiguousarray(np.asarray(t, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _pads(padding):
    """(left, right) zeros around the signal from an int or a (left, right) pair."""
    if isinstance(padding, (tuple, list)):
        return int(padding[0]), int(padding[1])
    return int(padding), int(padding)


class Oracle:
    """ctypes front of one build of ``dcn1d_oracle.c``."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_out_length.restype = _i64
        lib.oracle_out_length.argtypes = [_i64] * 5
        lib.oracle_forward.restype = _int
        lib.oracle_out_length_lr.restype = _i64
        lib.oracle_out_length_lr.argtypes = [_i64] * 6
        lib.oracle_forward.argtypes = [_p] * 5 + [_i64] * 12 + [_int, _p]
        lib.oracle_forward_points.restype = _int
        lib.oracle_forward_points.argtypes = [_p] * 5 + [_i64] * 12 + [_int, _p, _i64, _p]
        lib.oracle_sample_index.restype = _int
        lib.oracle_sample_index.argtypes = [_p] + [_i64] * 8 + [_int, _p, _p]
        lib.oracle_backward.restype = _int
        lib.oracle_backward.argtypes = [_p] * 5 + [_i64] * 12 + [_int] + [_p] * 5
        lib.oracle_threads.restype = _int
        lib.oracle_packed_trunk.argtypes = [_p] * 7 + [_i64] * 10 + [_p, _p]
        lib.oracle_packed_trunk.restype = _int
        lib.oracle_threads.argtypes = []
        lib.oracle_set_threads.restype = None
        lib.oracle_set_threads.argtypes = [_int]
        self.lib = lib
        self.path = lib_path

    def out_length(self, L_in: int, K: int, stride: int, padding, dilation: int) -> int:
        """Output length by the conv1d closed form; -1 when invalid.  ``padding`` is an int
        (both sides) or a (left, right) pair."""
        pl, pr = _pads(padding)
        return int(self.lib.oracle_out_length_lr(L_in, K, stride, pl, pr, dilation))

    def threads(self) -> int:
        return int(self.lib.oracle_threads())

    def set_threads(self, n: int) -> None:
        self.lib.oracle_set_threads(int(n))

    @staticmethod
    def _dims(x, weight, offsets, stride, padding, dilation, groups, offset_groups):
        B, C_in, L_in = x.shape
        C_out, _, K = weight.shape
        L_out = offsets.shape[2]
        if offsets.shape[1] != offset_groups:
            raise ValueError("offsets.shape[1] must equal offset_groups")
        if weight.shape[1] * groups != C_in or offsets.shape[3] != K or offsets.shape[0] != B:
            raise ValueError("weight/offsets shapes disagree with x and groups")
        pl, pr = _pads(padding)
        return (B, C_in, L_in, C_out, K, L_out, stride, pl, pr, dilation, groups, offset_groups)

    def forward(self, x, offsets, mask, weight, bias, stride, padding, dilation, groups,
                offset_groups, unconstrained) -> np.ndarray:
        """All outputs, float64 [B, C_out, L_out]."""
        xs, os_, ms, ws, bs = (_f32(t) for t in (x, offsets, mask, weight, bias))
        dims = self._dims(xs, ws, os_, stride, padding, dilation, groups, offset_groups)
        out = np.empty((dims[0], dims[3], dims[5]), dtype=np.float64)
        rc = self.lib.oracle_forward(_ptr(xs), _ptr(os_), _ptr(ms), _ptr(ws), _ptr(bs), *dims,
                                     int(bool(unconstrained)), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_forward rejected the shapes (code {rc})")
        return out

    def forward_points(self, x, offsets, mask, weight, bias, stride, padding, dilation, groups,
                       offset_groups, unconstrained, points) -> np.ndarray:
        """Selected outputs; ``points`` is an int array [n, 3] of (b, co, l)."""
        xs, os_, ms, ws, bs = (_f32(t) for t in (x, offsets, mask, weight, bias))
        dims = self._dims(xs, ws, os_, stride, padding, dilation, groups, offset_groups)
        pts = np.ascontiguousarray(np.asarray(points, dtype=np.int64).reshape(-1, 3))
        out = np.empty(pts.shape[0], dtype=np.float64)
        rc = self.lib.oracle_forward_points(_ptr(xs), _ptr(os_), _ptr(ms), _ptr(ws), _ptr(bs),
                                            *dims, int(bool(unconstrained)), _ptr(pts),
                                            pts.shape[0], _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_forward_points rejected the arguments (code {rc})")
        return out

    def backward(self, x, offsets, mask, weight, grad_out, stride, padding, dilation, groups,
                 offset_groups, unconstrained) -> dict:
        """Gradients of sum(grad_out * forward) as float64 arrays: grad_x, grad_offsets,
        grad_mask (None without a mask), grad_weight, grad_bias."""
        xs, os_, ms, ws, gs = (_f32(t) for t in (x, offsets, mask, weight, grad_out))
        dims = self._dims(xs, ws, os_, stride, padding, dilation, groups, offset_groups)
        if gs.shape != (dims[0], dims[3], dims[5]):
            raise ValueError("grad_out must be [B, C_out, L_out]")
        g = {"grad_x": np.empty(xs.shape, dtype=np.float64),
             "grad_offsets": np.empty(os_.shape, dtype=np.float64),
             "grad_mask": np.empty(os_.shape, dtype=np.float64) if ms is not None else None,
             "grad_weight": np.empty(ws.shape, dtype=np.float64),
             "grad_bias": np.empty(ws.shape[0], dtype=np.float64)}
        rc = self.lib.oracle_backward(_ptr(xs), _ptr(os_), _ptr(ms), _ptr(ws), _ptr(gs), *dims,
                                      int(bool(unconstrained)), _ptr(g["grad_x"]),
                                      _ptr(g["grad_offsets"]), _ptr(g["grad_mask"]),
                                      _ptr(g["grad_weight"]), _ptr(g["grad_bias"]))
        if rc != 0:
            raise ValueError(f"oracle_backward rejected the shapes (code {rc})")
        return g

    def packed_trunk(self, x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                     kernel_size, stride, padding, dilation, offset_groups):
        """PackedDeformConv1d's predicted offsets (and mask, None without a mask branch),
        float64 [B, offset_groups, L_out, K].  dw_weight is [C_in, 1, K] (or [C_in, K]);
        off_weight and mask_weight are [offset_groups*K, C_in] (or with a trailing 1)."""
        xs, dws, dbs, ows, obs, mws, mbs = (_f32(t) for t in (x, dw_weight, dw_bias, off_weight,
                                                              off_bias, mask_weight, mask_bias))
        B, C_in, L_in = xs.shape
        K = int(kernel_size)
        pl, pr = _pads(padding)
        if dws.size != C_in * K or ows.size != offset_groups * K * C_in:
            raise ValueError("trunk weight shapes disagree with C_in, K and offset_groups")
        if mws is not None and mws.size != ows.size:
            raise ValueError("mask_weight must have off_weight's shape")
        L_out = self.out_length(L_in, K, stride, (pl, pr), dilation)
        off = np.empty((B, offset_groups, L_out, K), dtype=np.float64)
        mask = np.empty_like(off) if mws is not None else None
        rc = self.lib.oracle_packed_trunk(_ptr(xs), _ptr(dws), _ptr(dbs), _ptr(ows), _ptr(obs),
                                          _ptr(mws), _ptr(mbs), B, C_in, L_in, K, L_out, stride,
                                          pl, pr, dilation, offset_groups, _ptr(off), _ptr(mask))
        if rc != 0:
            raise ValueError(f"oracle_packed_trunk rejected the arguments (code {rc})")
        return off, mask

    def packed_forward(self, x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                       weight, bias, stride, padding, dilation, groups, offset_groups,
                       unconstrained, dtype=None):
        """PackedDeformConv1d's output: the trunk's offsets (and mask), rounded to ``dtype``
        (x's own dtype by default: the tensor the layer passes on), then the forward.
        Returns (out float64, offsets float64, mask float64 or None), the latter two
        before that rounding."""
        K = weight.shape[2]
        off, mask = self.packed_trunk(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight,
                                      mask_bias, K, stride, padding, dilation, offset_groups)
        dt = dtype if dtype is not None else (x.dtype if isinstance(x, torch.Tensor)
                                              else torch.float32)
        off_r = torch.from_numpy(off).to(dt)
        mask_r = torch.from_numpy(mask).to(dt) if mask is not None else None
        out = self.forward(x, off_r, mask_r, weight, bias, stride, padding, dilation, groups,
                           offset_groups, unconstrained)
        return out, off, mask

    def sample_index(self, offsets, L_in, K, stride, padding, dilation, unconstrained):
        """(i0 int32, frac float32) for every tap, each shaped like ``offsets``."""
        os_ = _f32(offsets)
        B, G, L_out, K2 = os_.shape
        if K2 != K:
            raise ValueError("offsets.shape[3] must equal K")
        i0 = np.empty(os_.shape, dtype=np.int32)
        fr = np.empty(os_.shape, dtype=np.float32)
        rc = self.lib.oracle_sample_index(_ptr(os_), B, G, L_in, K, L_out, stride, padding,
                                          dilation, int(bool(unconstrained)), _ptr(i0), _ptr(fr))
        if rc != 0:
            raise ValueError("oracle_sample_index: offsets length disagrees with the closed form")
        return i0, fr


_default = None
_lock = threading.Lock()


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(_build.build())
    return _default


def out_length(*a):
    return get().out_length(*a)


def forward(*a, **k):
    return get().forward(*a, **k)


def forward_points(*a, **k):
    return get().forward_points(*a, **k)


def sample_index(*a, **k):
    return get().sample_index(*a, **k)


def backward(*a, **k):
    return get().backward(*a, **k)


def packed_trunk(*a, **k):
    return get().packed_trunk(*a, **k)


def packed_forward(*a, **k):
    return get().packed_forward(*a, **k)


def threads():
    return get().threads()


def set_threads(n):
    return get().set_threads(n)
