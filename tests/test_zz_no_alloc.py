"""dcn1d_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (a loop that must not allocate, a runtime that owns every allocation) get the
library's fixed 48 MiB static scratch instead of a workspace.  These tests call that entry
point through the C ABI and compare it with the workspace entry point (dcn1d_forward_ws,
scratch from torch) on the same inputs, twice in a row with different inputs, so the second
call also shows that the scratch left over from the first does not leak into the result.
This file is named to be collected last.
"""
import ctypes

import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from deformable_convolution_dcn1d_b200._binding import _desc, _ref

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4   # the normwise bound the other fp32 GPU tests use


def _noalloc_through_c_abi(w, td, out):
    lib = dcn.load()
    descs = [_desc(t) for t in (td["x"], td["offsets"], td["mask"], td["weight"], td["bias"], out)]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.dcn1d_forward_noalloc(*(_ref(d) for d in descs[:5]), w.stride, w.padding,
                                     w.dilation, w.groups, w.offset_groups,
                                     int(w.unconstrained), _ref(descs[5]),
                                     ctypes.c_void_p(stream))


def _norm_err(a, b):
    return (a.double() - b.double()).abs().max().item() / b.double().abs().max().item()


def test_noalloc_matches_workspace_entry_on_two_calls():
    w = W.USAGE_F32   # the dc1d page's usage shape in fp32: the path that needs scratch
    assert torch.cuda.is_available()
    for seed in (0, 1):
        td = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w, seed).items()}
        assert dcn.dcn1d_forward_workspace_size(td["x"], td["offsets"], td["mask"], td["weight"],
                                                td["bias"], w.stride, w.padding, w.dilation,
                                                w.groups, w.offset_groups,
                                                w.unconstrained) > 0
        ref = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"],
                                w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                                w.unconstrained)
        out = torch.full_like(ref, float("nan"))
        st = _noalloc_through_c_abi(w, td, out)
        assert st == 0, dcn.dcn1d_status_string(st)
        assert dcn.dcn1d_last_launch_count() >= 2   # the scratch-using tensor-core path ran
        torch.cuda.synchronize()
        assert dcn.dcn1d_device_status() == 0
        assert torch.isfinite(out).all()
        assert _norm_err(out, ref) <= TOL_F32, seed


def test_noalloc_rejects_scratch_past_its_limit():
    # C_in = C_out = 1024, K = 16: the split weight alone is 128 MiB > 48 MiB.
    B, C, K, L = 1, 1024, 16, 128
    L_out = oracle.out_length(L, K, 1, 0, 1)
    x = torch.zeros(B, C, L, device="cuda")
    off = torch.zeros(B, 1, L_out, K, device="cuda")
    wgt = torch.zeros(C, C, K, device="cuda")
    out = torch.full((B, C, L_out), float("nan"), device="cuda")
    with pytest.raises(dcn.Dcn1dError) as e:
        dcn.dcn1d_forward_noalloc(x, off, None, wgt, None, 1, 0, 1, 1, 1, False, out=out)
    assert e.value.status == 5   # DCN1D_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.isnan(out).all()   # nothing was launched
