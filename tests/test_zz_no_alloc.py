"""dcn1d_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (a loop that must not allocate, a runtime that owns every allocation) get the
library's fixed 48 MiB static scratch instead of a workspace wherever a path needs scratch.
No forward path needs any now (the fp32 tensor-core path forms the weight's low part and
adds its split-K partial sums on chip), so the entry point runs every valid argument set as
dcn1d_forward.  These tests call it through the C ABI and compare it with dcn1d_forward on
the same inputs, twice in a row with different inputs, and on a shape whose fp32 path once
needed more scratch than the array holds.  This file is named to be collected last.
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


def test_noalloc_matches_forward_on_two_calls():
    w = W.USAGE_F32   # the dc1d page's usage shape in fp32 (split-K tensor-core path)
    assert torch.cuda.is_available()
    for seed in (0, 1):
        td = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w, seed).items()}
        assert dcn.dcn1d_forward_workspace_size(td["x"], td["offsets"], td["mask"], td["weight"],
                                                td["bias"], w.stride, w.padding, w.dilation,
                                                w.groups, w.offset_groups,
                                                w.unconstrained) == 0
        ref = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"],
                                w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                                w.unconstrained)
        out = torch.full_like(ref, float("nan"))
        st = _noalloc_through_c_abi(w, td, out)
        assert st == 0, dcn.dcn1d_status_string(st)
        assert dcn.dcn1d_last_launch_count() == 1   # the one-launch tensor-core path ran
        torch.cuda.synchronize()
        assert dcn.dcn1d_device_status() == 0
        assert torch.equal(out.view(torch.int32), ref.view(torch.int32)), seed
        r = oracle.forward(*[None if td[k] is None else td[k][:1].cpu() if k in
                             ("x", "offsets", "mask") else td[k].cpu()
                             for k in ("x", "offsets", "mask", "weight", "bias")],
                           w.stride, (w.padding, w.padding), w.dilation, w.groups,
                           w.offset_groups, w.unconstrained)
        assert _norm_err(out[:1].cpu(), torch.from_numpy(r)) <= TOL_F32, seed


def test_noalloc_runs_a_shape_past_the_old_scratch_limit():
    # C_in = C_out = 1024, K = 16: a low tf32 weight part in memory alone would be
    # 64 MiB > 48 MiB; the on-chip form needs none, so the call runs (split-K cluster).
    B, C, K, L = 1, 1024, 16, 128
    L_out = oracle.out_length(L, K, 1, 0, 1)
    gen = torch.Generator().manual_seed(7)
    x = torch.randn(B, C, L, generator=gen).cuda()
    off = (torch.rand(B, 1, L_out, K, generator=gen) * 4 - 2).cuda()
    wgt = (torch.randn(C, C, K, generator=gen) / 128).cuda()
    out = torch.full((B, C, L_out), float("nan"), device="cuda")
    dcn.dcn1d_forward_noalloc(x, off, None, wgt, None, 1, 0, 1, 1, 1, False, out=out)
    ref = dcn.dcn1d_forward(x, off, None, wgt, None, 1, 0, 1, 1, 1, False)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    r = oracle.forward(x[:, :, :].cpu(), off.cpu(), None, wgt.cpu(), None, 1, (0, 0), 1, 1, 1,
                       False)
    assert _norm_err(out.cpu(), torch.from_numpy(r)) <= TOL_F32
