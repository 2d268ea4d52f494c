"""ctypes binding of libdcn1d.so (include/dcn1d.h).

Argument marshalling only: torch tensors are described to the C ABI by their
device pointer, dtype and shape, and the current torch CUDA stream is passed
through.  Every step of the forward runs in the library's CUDA kernels; there
is no Python or CPU fallback, and a missing or unbuildable library raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

from . import build as _build

_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int
_P = ctypes.c_void_p

DCN1D_F32 = 0
DCN1D_BF16 = 1
DCN1D_F16 = 2
_DTYPES = {torch.float32: DCN1D_F32, torch.bfloat16: DCN1D_BF16, torch.float16: DCN1D_F16}
_BAD_DTYPE = 99   # any other torch dtype: the library rejects it with DCN1D_ERR_DTYPE

STATUS = {0: "DCN1D_OK", 1: "DCN1D_ERR_NULL", 2: "DCN1D_ERR_DTYPE", 3: "DCN1D_ERR_SHAPE",
          4: "DCN1D_ERR_ARG", 5: "DCN1D_ERR_UNSUPPORTED", 6: "DCN1D_ERR_LAUNCH",
          7: "DCN1D_ERR_TIMEOUT", 8: "DCN1D_ERR_CUDA"}


class Dcn1dTensor(ctypes.Structure):
    _fields_ = [("data", _P), ("dtype", _I32), ("ndim", _I32), ("shape", _I64 * 4)]


_SHAPE4 = _I64 * 4


class Dcn1dError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dcn1d_status_string(status)} ({status})")


_lib = None
_lock = threading.Lock()

# Exported symbols and their signatures: (name, restype, argtypes).
_T = ctypes.POINTER(Dcn1dTensor)
SIGNATURES = [
    ("dcn1d_out_length", _I64, [_I64] * 5),
    ("dcn1d_forward", _INT, [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _P]),
    ("dcn1d_status_string", ctypes.c_char_p, [_INT]),
    ("dcn1d_sample_index", _INT, [_T, _I64, _I64, _I64, _I64, _INT, _P, _P, _P]),
    ("dcn1d_forward_kernel_name", ctypes.c_char_p,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T]),
    ("dcn1d_last_launch_count", _INT, []),
    ("dcn1d_device_status", _INT, [_P]),
    ("dcn1d_forward_workspace_size", _I64,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T]),
    ("dcn1d_forward_ws", _INT,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _P, ctypes.c_size_t, _P]),
    ("dcn1d_set_timing_events", None, [_P, _P]),
    ("dcn1d_forward_noalloc", _INT,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _P]),
    ("dcn1d_backward_workspace_size", _I64,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _T, _T, _T, _T]),
    ("dcn1d_backward", _INT,
     [_T, _T, _T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _T, _T, _T, _T, _P,
      ctypes.c_size_t, _P]),
    ("dcn1d_out_length_lr", _I64, [_I64] * 6),
    ("dcn1d_forward_lr_kernel_name", ctypes.c_char_p, [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT, _T]),
    ("dcn1d_forward_lr", _INT,
     [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT, _T, _P, ctypes.c_size_t, _P]),
    ("dcn1d_forward_lr_workspace_size", _I64, [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT, _T]),
    ("dcn1d_backward_lr_workspace_size", _I64,
     [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT] + [_T] * 5),
    ("dcn1d_backward_lr", _INT,
     [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT] + [_T] * 5 + [_P, ctypes.c_size_t, _P]),
    ("dcn1d_packed_trunk", _INT, [_T] * 7 + [_I64] * 5 + [_T, _T, _P]),
    ("dcn1d_packed_trunk_kernel_name", ctypes.c_char_p, [_T] * 7 + [_I64] * 5 + [_T, _T]),
    ("dcn1d_packed_forward_workspace_size", _I64,
     [_T] * 9 + [_I64] * 6 + [_INT] + [_T] * 3),
    ("dcn1d_packed_forward", _INT,
     [_T] * 9 + [_I64] * 6 + [_INT] + [_T] * 3 + [_P, ctypes.c_size_t, _P]),
    ("dcn1d_packed_forward_kernel_name", ctypes.c_char_p,
     [_T] * 9 + [_I64] * 6 + [_INT] + [_T] * 3),
    ("dcn1d_backward_kernel_name", ctypes.c_char_p,
     [_T, _T, _T, _T, _T] + [_I64] * 6 + [_INT] + [_T] * 5),
    ("dcn1d_test_forward_stalled", _INT,
     [_T, _T, _T, _I64, _I64, _I64, _I64, _I64, _INT, _T, _I64, _P]),
]


def resolve_padding(padding, kernel_size, stride=1, dilation=1):
    """(left, right) zeros around the signal from an int (both sides), a (left, right)
    pair, "valid" (none) or "same" (stride 1: dilation*(kernel_size-1) // 2 on the left,
    the rest on the right, so that L_out = L_in -- nn.Conv1d's reading, which the dc1d
    page's output-length rule follows)."""
    if isinstance(padding, str):
        if padding == "valid":
            return 0, 0
        if padding == "same":
            if stride != 1:
                raise ValueError('padding="same" needs stride 1')
            tot = dilation * (kernel_size - 1)
            return tot // 2, tot - tot // 2
        raise ValueError(f"unknown padding {padding!r}")
    if isinstance(padding, (tuple, list)):
        if len(padding) != 2:
            raise ValueError("padding pair must be (left, right)")
        return int(padding[0]), int(padding[1])
    return int(padding), int(padding)


def lib_path() -> str:
    return _build.LIB


def load():
    """Load libdcn1d.so, building it from csrc/ with nvcc if it is missing or stale."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            if not os.path.exists(path):
                raise ImportError(f"libdcn1d.so not found at {path}")
            lib = ctypes.CDLL(path)
            for name, res, args in SIGNATURES:
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _desc(t):
    """dcn1d_tensor describing a contiguous torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if t.ndim > 4:
        raise ValueError("at most 4 dimensions")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    shape = t.shape
    return Dcn1dTensor(t.data_ptr() if t.numel() > 0 else None,
                       _DTYPES.get(t.dtype, _BAD_DTYPE), len(shape), _SHAPE4(*shape))


def _ref(d):
    return None if d is None else ctypes.byref(d)


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _check_device(tensors):
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("every tensor must be on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("every tensor must be on the same CUDA device")
    return dev


def dcn1d_out_length(L_in: int, kernel_size: int, stride: int = 1, padding=0,
                     dilation: int = 1) -> int:
    """Output length (-1 when invalid); ``padding`` as in resolve_padding."""
    pl, pr = resolve_padding(padding, kernel_size, stride, dilation)
    return int(load().dcn1d_out_length_lr(L_in, kernel_size, stride, pl, pr, dilation))


def dcn1d_status_string(status: int) -> str:
    return load().dcn1d_status_string(int(status)).decode()


def dcn1d_last_launch_count() -> int:
    return int(load().dcn1d_last_launch_count())


def dcn1d_set_timing_events(begin, end) -> None:
    """The next forward on this thread records these torch.cuda.Events around its main kernel."""
    load().dcn1d_set_timing_events(_P(begin.cuda_event if begin is not None else None),
                                   _P(end.cuda_event if end is not None else None))


def dcn1d_device_status(stream=None, device=None) -> int:
    """Synchronise ``stream`` and return (and clear) the kernels' bounded-wait status:
    0 (DCN1D_OK) or 7 (DCN1D_ERR_TIMEOUT)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    lib = load()
    with torch.cuda.device(dev):
        return int(lib.dcn1d_device_status(_P(_stream_ptr(stream, dev))))


def _out_for(x, weight, offsets):
    L_out = offsets.shape[2] if offsets.ndim == 4 else 0
    return torch.empty((x.shape[0], weight.shape[0], L_out), dtype=x.dtype, device=x.device)


def dcn1d_forward(x, offsets, mask, weight, bias, stride=1, padding=0, dilation=1, groups=1,
                  offset_groups=1, unconstrained=False, out=None, stream=None, workspace=None):
    """Deformable conv1d forward through the C ABI; returns ``out`` [B, C_out, L_out].

    x [B, C_in, L_in]; offsets and mask [B, offset_groups, L_out, K] (mask may be None);
    weight [C_out, C_in/groups, K]; bias [C_out] or None.  All CUDA, contiguous, one dtype
    (float32, bfloat16 or float16).  ``padding``: an int, a (left, right) pair, "valid" or "same"
    (see resolve_padding).  ``out`` is allocated with torch when not given.  Scratch that a
    path needs (``dcn1d_forward_workspace_size``; no present path needs any) is allocated
    with torch unless a uint8 CUDA tensor ``workspace`` is given; ``workspace=False`` passes
    none.  Without ``workspace`` such scratch is kept for later calls on the same device and
    stream (see clear_workspace_cache).  Runs on ``stream`` (default: the current torch
    stream of x's device); does not synchronise.
    """
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    dev = _check_device((x, offsets, mask, weight, bias, out))
    if out is None:
        out = _out_for(x, weight, offsets)
    tensors = (x, offsets, mask, weight, bias, out)
    refs = [_ref(_desc(t)) for t in tensors]
    lib = load()
    args = (stride, pl, pr, dilation, groups, offset_groups, int(bool(unconstrained)))
    ctx = (contextlib.nullcontext() if torch.cuda.current_device() == dev.index
           else torch.cuda.device(dev))
    with ctx:
        sptr = _stream_ptr(stream, dev)
        ws_ptr, ws_bytes = None, 0
        if workspace is not False:
            key = (dev.index, args, tuple(None if t is None else
                                          (tuple(t.shape), t.dtype, t.data_ptr() % 256)
                                          for t in tensors))
            need = _need_cache.get(key)
            if need is None:
                need = int(lib.dcn1d_forward_lr_workspace_size(*refs[:5], *args, refs[5]))
                if need < 0:
                    raise Dcn1dError(-need, "dcn1d_forward_workspace_size")
                if len(_need_cache) > 4096:
                    _need_cache.clear()
                _need_cache[key] = need
            if need > 0:
                if workspace is None:
                    workspace = _ws_cache.get((dev.index, sptr))
                    if workspace is None or workspace.numel() < need:
                        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
                        if isinstance(stream, torch.cuda.Stream):
                            workspace.record_stream(stream)
                        _ws_cache[(dev.index, sptr)] = workspace
                if workspace.numel() < need or workspace.dtype != torch.uint8:
                    raise ValueError(f"workspace must be a uint8 tensor of >= {need} bytes")
                ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        st = lib.dcn1d_forward_lr(*refs[:5], *args, refs[5], _P(ws_ptr), ws_bytes, _P(sptr))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_forward")
    return out


# Scratch reused by dcn1d_forward calls that pass no workspace: one uint8 tensor per
# (device, stream), grown when a call needs more (calls on one stream run in order, so
# they can share it); and the scratch size of each call signature seen.
_ws_cache = {}
_need_cache = {}


def clear_workspace_cache() -> None:
    """Drop the scratch tensors dcn1d_forward keeps between calls."""
    _ws_cache.clear()
    _need_cache.clear()


GRADS = ("x", "offsets", "mask", "weight", "bias")


def dcn1d_backward(x, offsets, mask, weight, grad_out, stride=1, padding=0, dilation=1,
                   groups=1, offset_groups=1, unconstrained=False, wanted=GRADS, grads=None,
                   workspace=None, stream=None):
    """Gradients of sum(grad_out * forward) through the C ABI.

    Returns a dict {name: tensor} for the names in ``wanted`` (a subset of "x", "offsets",
    "mask", "weight", "bias"; "mask" only when a mask is given), each shaped like its
    input (bias: [C_out]) in the inputs' dtype.  ``grads`` may supply some of those
    tensors (they are overwritten); the rest, and the scratch the call needs, are
    allocated with torch unless a uint8 CUDA tensor ``workspace`` is given.  Runs on
    ``stream``; does not synchronise.
    """
    wanted = tuple(n for n in wanted if n != "mask" or mask is not None)
    unknown = set(wanted) - set(GRADS)
    if unknown:
        raise ValueError(f"unknown gradients {sorted(unknown)}")
    dev = _check_device((x, offsets, mask, weight, grad_out))
    like = {"x": x, "offsets": offsets, "mask": mask, "weight": weight}
    out = dict(grads or {})
    for n in wanted:
        if n not in out:
            shape = (weight.shape[0],) if n == "bias" else like[n].shape
            out[n] = torch.empty(shape, dtype=x.dtype, device=dev)
    ins = [_desc(t) for t in (x, offsets, mask, weight, grad_out)]
    gd = [_desc(out.get(n)) for n in GRADS]
    lib = load()
    refs = [_ref(d) for d in ins] + [_ref(d) for d in gd]
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    args = (stride, pl, pr, dilation, groups, offset_groups, int(bool(unconstrained)))
    with torch.cuda.device(dev):
        need = int(lib.dcn1d_backward_lr_workspace_size(*refs[:5], *args, *refs[5:]))
        if need < 0:
            raise Dcn1dError(-need, "dcn1d_backward_workspace_size")
        ws_ptr, ws_bytes = None, 0
        if need > 0:
            if workspace is None:
                workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            if workspace.numel() < need or workspace.dtype != torch.uint8:
                raise ValueError(f"workspace must be a uint8 tensor of >= {need} bytes")
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        st = lib.dcn1d_backward_lr(*refs[:5], *args, *refs[5:], _P(ws_ptr), ws_bytes,
                                   _P(_stream_ptr(stream, dev)))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_backward")
    return {n: out[n] for n in wanted}


def dcn1d_backward_kernel_name(x, offsets, mask, weight, grad_out, stride=1, padding=0,
                               dilation=1, groups=1, offset_groups=1, unconstrained=False,
                               wanted=GRADS):
    """Which contraction kernels dcn1d_backward runs ("tcgen05_gemm" or "cuda_core_gemm")."""
    wanted = tuple(n for n in wanted if n != "mask" or mask is not None)
    like = {"x": x, "offsets": offsets, "mask": mask, "weight": weight}
    probe = {n: torch.empty((weight.shape[0],) if n == "bias" else like[n].shape,
                            dtype=x.dtype, device="meta") for n in wanted}
    gd = [None if probe.get(n) is None else _meta_desc(probe[n]) for n in GRADS]
    ins = [_desc(t) if t is None or t.device.type != "meta" else _meta_desc(t)
           for t in (x, offsets, mask, weight, grad_out)]
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    r = load().dcn1d_backward_kernel_name(*(_ref(d) for d in ins), stride, pl, pr, dilation,
                                          groups, offset_groups, int(bool(unconstrained)),
                                          *(_ref(d) for d in gd))
    return None if r is None else r.decode()


def dcn1d_backward_workspace_size(x, offsets, mask, weight, grad_out, stride=1, padding=0,
                                  dilation=1, groups=1, offset_groups=1, unconstrained=False,
                                  wanted=GRADS) -> int:
    """Bytes of scratch dcn1d_backward needs for these arguments and wanted gradients."""
    wanted = tuple(n for n in wanted if n != "mask" or mask is not None)
    like = {"x": x, "offsets": offsets, "mask": mask, "weight": weight}
    probe = {n: torch.empty((weight.shape[0],) if n == "bias" else like[n].shape,
                            dtype=x.dtype, device="meta") for n in wanted}
    gd = [None if probe.get(n) is None else _meta_desc(probe[n]) for n in GRADS]
    ins = [_desc(t) for t in (x, offsets, mask, weight, grad_out)]
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    need = int(load().dcn1d_backward_lr_workspace_size(
        *(_ref(d) for d in ins), stride, pl, pr, dilation, groups, offset_groups,
        int(bool(unconstrained)), *(_ref(d) for d in gd)))
    if need < 0:
        raise Dcn1dError(-need, "dcn1d_backward_workspace_size")
    return need


def dcn1d_forward_noalloc(x, offsets, mask, weight, bias, stride=1, padding=0, dilation=1,
                          groups=1, offset_groups=1, unconstrained=False, out=None, stream=None):
    """The forward for callers that cannot allocate device memory: the library's own
    48 MiB static scratch instead of a workspace.  ``out`` must be given (this call
    allocates nothing).  Calls whose GPU work overlaps share the scratch and race."""
    if out is None:
        raise ValueError("dcn1d_forward_noalloc allocates nothing: pass out")
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    if pl != pr:
        raise ValueError("dcn1d_forward_noalloc takes symmetric padding only")
    padding = pl
    dev = _check_device((x, offsets, mask, weight, bias, out))
    descs = [_desc(t) for t in (x, offsets, mask, weight, bias, out)]
    lib = load()
    with torch.cuda.device(dev):
        st = lib.dcn1d_forward_noalloc(*(_ref(d) for d in descs[:5]), stride, padding,
                                       dilation, groups, offset_groups,
                                       int(bool(unconstrained)), _ref(descs[5]),
                                       _P(_stream_ptr(stream, dev)))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_forward_noalloc")
    return out


def dcn1d_test_forward_stalled(x, offsets, weight, stride=1, padding=0, dilation=1, groups=1,
                               offset_groups=1, unconstrained=False, out=None,
                               wait_limit_ns=1_000_000, stream=None):
    """Test hook of the failure path (include/dcn1d.h): the bf16 tensor-core kernel with its
    loader switched off and a short wait limit.  Returns the call's status code (no raise);
    the timeout itself is reported by the next dcn1d_device_status()."""
    dev = _check_device((x, offsets, weight, out))
    if out is None:
        out = _out_for(x, weight, offsets)
    descs = [_desc(t) for t in (x, offsets, weight, out)]
    with torch.cuda.device(dev):
        return int(load().dcn1d_test_forward_stalled(
            _ref(descs[0]), _ref(descs[1]), _ref(descs[2]), stride, int(padding), dilation,
            groups, offset_groups, int(bool(unconstrained)), _ref(descs[3]), int(wait_limit_ns),
            _P(_stream_ptr(stream, dev))))


def dcn1d_forward_workspace_size(x, offsets, mask, weight, bias, stride=1, padding=0,
                                 dilation=1, groups=1, offset_groups=1, unconstrained=False,
                                 out=None) -> int:
    """Bytes of scratch the fastest path needs for these arguments (0 if none)."""
    if out is None:
        out = _out_for(x, weight, offsets)
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    descs = [_desc(t) for t in (x, offsets, mask, weight, bias, out)]
    need = int(load().dcn1d_forward_lr_workspace_size(*(_ref(d) for d in descs[:5]), stride,
                                                      pl, pr, dilation, groups, offset_groups,
                                                      int(bool(unconstrained)),
                                                      _ref(descs[5])))
    if need < 0:
        raise Dcn1dError(-need, "dcn1d_forward_workspace_size")
    return need


def dcn1d_forward_kernel_name(x, offsets, mask, weight, bias, stride=1, padding=0, dilation=1,
                              groups=1, offset_groups=1, unconstrained=False, out=None):
    """Name of the kernel dcn1d_forward would launch, or None for invalid arguments."""
    pl, pr = resolve_padding(padding, weight.shape[2], stride, dilation)
    if out is None:
        out = torch.empty((x.shape[0], weight.shape[0], offsets.shape[2]), dtype=x.dtype,
                          device="meta")
    descs = [_desc(t) if t is None or t.device.type != "meta" else _meta_desc(t)
             for t in (x, offsets, mask, weight, bias, out)]
    r = load().dcn1d_forward_lr_kernel_name(*(_ref(d) for d in descs[:5]), stride, pl, pr,
                                            dilation, groups, offset_groups,
                                            int(bool(unconstrained)), _ref(descs[5]))
    return None if r is None else r.decode()


def _meta_desc(t):
    d = Dcn1dTensor()
    d.data = 16 if t.numel() > 0 else None    # a non-NULL placeholder; never dereferenced
    d.dtype = _DTYPES.get(t.dtype, _BAD_DTYPE)
    d.ndim = t.ndim
    for i, s in enumerate(t.shape):
        d.shape[i] = s
    return d


def dcn1d_sample_index(offsets, L_in, stride=1, padding=0, dilation=1, unconstrained=False,
                       stream=None):
    """(i0 int32, frac float32) of every tap of ``offsets``, computed on the GPU."""
    dev = _check_device((offsets,))
    i0 = torch.empty(offsets.shape, dtype=torch.int32, device=dev)
    fr = torch.empty(offsets.shape, dtype=torch.float32, device=dev)
    d = _desc(offsets)
    lib = load()
    with torch.cuda.device(dev):
        st = lib.dcn1d_sample_index(ctypes.byref(d), L_in, stride, padding, dilation,
                                    int(bool(unconstrained)), _P(i0.data_ptr()),
                                    _P(fr.data_ptr()), _P(_stream_ptr(stream, dev)))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_sample_index")
    return i0, fr


# ------------------------------------------------------------------ PackedDeformConv1d


def _trunk_outputs(x, dw_weight, mask_weight, stride, pl, pr, dilation, offset_groups):
    K = dw_weight.shape[2]
    L_out = int(load().dcn1d_out_length_lr(x.shape[2], K, stride, pl, pr, dilation))
    shape = (x.shape[0], offset_groups, max(L_out, 0), K)
    off = torch.empty(shape, dtype=x.dtype, device=x.device)
    mask = torch.empty(shape, dtype=x.dtype, device=x.device) if mask_weight is not None else None
    return off, mask


def dcn1d_packed_trunk(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight=None,
                       mask_bias=None, stride=1, padding=0, dilation=1, offset_groups=1,
                       offsets_out=None, mask_out=None, stream=None):
    """PackedDeformConv1d's offset (and mask) predictor through the C ABI.

    x [B, C_in, L_in]; dw_weight [C_in, 1, K] and dw_bias [C_in] (the depthwise trunk);
    off_weight [offset_groups*K, C_in(, 1)] and off_bias (the offset head); mask_weight and
    mask_bias likewise for the sigmoid mask head, or None.  Returns (offsets, mask) as
    [B, offset_groups, L_out, K] tensors (mask None without a mask head).  Does not
    synchronise.
    """
    K = dw_weight.shape[2]
    pl, pr = resolve_padding(padding, K, stride, dilation)
    dev = _check_device((x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                         offsets_out, mask_out))
    if offsets_out is None or (mask_weight is not None and mask_out is None):
        o, m = _trunk_outputs(x, dw_weight, mask_weight, stride, pl, pr, dilation,
                              offset_groups)
        offsets_out = o if offsets_out is None else offsets_out
        mask_out = m if mask_out is None else mask_out
    tensors = (x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
               offsets_out, mask_out)
    refs = [_ref(_desc(t)) for t in tensors]
    lib = load()
    with torch.cuda.device(dev):
        st = lib.dcn1d_packed_trunk(*refs[:7], stride, pl, pr, dilation, offset_groups,
                                    refs[7], refs[8], _P(_stream_ptr(stream, dev)))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_packed_trunk")
    return offsets_out, mask_out


def dcn1d_packed_trunk_kernel_name(x, dw_weight, dw_bias, off_weight, off_bias,
                                   mask_weight=None, mask_bias=None, stride=1, padding=0,
                                   dilation=1, offset_groups=1):
    """Name of the trunk kernel these arguments select (None if invalid)."""
    K = dw_weight.shape[2]
    pl, pr = resolve_padding(padding, K, stride, dilation)
    o, m = _trunk_outputs(x, dw_weight, mask_weight, stride, pl, pr, dilation, offset_groups)
    tensors = (x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias, o, m)
    refs = [_ref(_desc(t)) for t in tensors]
    r = load().dcn1d_packed_trunk_kernel_name(*refs[:7], stride, pl, pr, dilation,
                                              offset_groups, refs[7], refs[8])
    return r.decode() if r else None


def dcn1d_packed_forward_kernel_name(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight,
                                     mask_bias, weight, bias, stride=1, padding=0, dilation=1,
                                     groups=1, offset_groups=1, unconstrained=False,
                                     with_offsets=False):
    """Which form dcn1d_packed_forward takes ("packed_fused_tcgen05", or "<trunk>+<forward>"
    for two launches); None for invalid arguments."""
    K = weight.shape[2]
    pl, pr = resolve_padding(padding, K, stride, dilation)
    off_t = mask_t = None
    if with_offsets:
        off_t, mask_t = _trunk_outputs(x, dw_weight, mask_weight, stride, pl, pr, dilation,
                                       offset_groups)
    L_out = int(load().dcn1d_out_length_lr(x.shape[2], K, stride, pl, pr, dilation))
    out = torch.empty((x.shape[0], weight.shape[0], max(L_out, 0)), dtype=x.dtype,
                      device="meta")
    tensors = (x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias, weight,
               bias, off_t, mask_t)
    descs = [_desc(t) if t is None or t.device.type != "meta" else _meta_desc(t)
             for t in tensors] + [_meta_desc(out)]
    r = load().dcn1d_packed_forward_kernel_name(*[_ref(d) for d in descs[:9]], stride, pl, pr,
                                                dilation, groups, offset_groups,
                                                int(bool(unconstrained)),
                                                *[_ref(d) for d in descs[9:]])
    return r.decode() if r else None


def dcn1d_packed_forward(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                         weight, bias, stride=1, padding=0, dilation=1, groups=1,
                         offset_groups=1, unconstrained=False, with_offsets=False, out=None,
                         stream=None, workspace=None):
    """PackedDeformConv1d's forward through the C ABI: the trunk predicts the offsets (and,
    with mask_weight, the sigmoid mask), then the deformable convolution runs with them.

    Returns ``out`` [B, C_out, L_out]; with ``with_offsets`` the dc1d page's forms:
    (out, offsets), or (out, (offsets, mask)) when the layer is modulated.  Without
    ``with_offsets`` the predicted tensors live in the call's workspace (a uint8 CUDA
    tensor of ``dcn1d_packed_forward_workspace_size`` bytes, allocated with torch and kept
    per device and stream when not given).  Does not synchronise.
    """
    K = weight.shape[2]
    pl, pr = resolve_padding(padding, K, stride, dilation)
    dev = _check_device((x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                         weight, bias, out))
    off_t = mask_t = None
    if with_offsets:
        off_t, mask_t = _trunk_outputs(x, dw_weight, mask_weight, stride, pl, pr, dilation,
                                       offset_groups)
    if out is None:
        L_out = int(load().dcn1d_out_length_lr(x.shape[2], K, stride, pl, pr, dilation))
        out = torch.empty((x.shape[0], weight.shape[0], max(L_out, 0)), dtype=x.dtype,
                          device=x.device)
    tensors = (x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias, weight,
               bias, off_t, mask_t, out)
    refs = [_ref(_desc(t)) for t in tensors]
    lib = load()
    args = (stride, pl, pr, dilation, groups, offset_groups, int(bool(unconstrained)))
    with torch.cuda.device(dev):
        sptr = _stream_ptr(stream, dev)
        need = int(lib.dcn1d_packed_forward_workspace_size(*refs[:9], *args, *refs[9:]))
        if need < 0:
            raise Dcn1dError(-need, "dcn1d_packed_forward_workspace_size")
        ws_ptr, ws_bytes = None, 0
        if need > 0:
            if workspace is None:
                key = ("packed", dev.index, sptr)
                workspace = _ws_cache.get(key)
                if workspace is None or workspace.numel() < need:
                    workspace = torch.empty(need, dtype=torch.uint8, device=dev)
                    if isinstance(stream, torch.cuda.Stream):
                        workspace.record_stream(stream)
                    _ws_cache[key] = workspace
            if workspace.dtype != torch.uint8 or workspace.numel() < need:
                raise ValueError(f"workspace must be a uint8 tensor of >= {need} bytes")
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        st = lib.dcn1d_packed_forward(*refs[:9], *args, *refs[9:], _P(ws_ptr), ws_bytes,
                                      _P(sptr))
    if st != 0:
        raise Dcn1dError(st, "dcn1d_packed_forward")
    if not with_offsets:
        return out
    return (out, (off_t, mask_t)) if mask_weight is not None else (out, off_t)
