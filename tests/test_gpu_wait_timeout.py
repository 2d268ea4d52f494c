"""The bounded waits of the tensor-core kernel give up, report and leave the GPU usable (GPU).

Every on-chip wait of the tensor-core kernels is bounded; a kernel whose wait runs out
records DCN1D_ERR_TIMEOUT in a device status word, drains what it issued, frees its tensor
memory and exits.  The test hook ``dcn1d_test_forward_stalled`` runs that kernel in a build
whose loader never issues a load, with a 1 ms limit: nothing faults, traps or hangs, the
call returns, the status reads DCN1D_ERR_TIMEOUT once, and an ordinary forward right after
it is correct with a clean status.
"""
import time

import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
from deformable_convolution_dcn1d_b200 import _binding as B
import oracle
import workloads as W
from gpu_util import TOL, gpu_forward, kernel_name, norm_err, oracle_full, to_dev

pytestmark = pytest.mark.gpu

DCN1D_ERR_TIMEOUT = 7


def _case():
    return W.small_case(3, B=2, C_in=64, C_out=128, K=3, stride=1, padding=1, dilation=1,
                        groups=1, offset_groups=1, L_in=512, L_out=512, dtype="bf16",
                        mask=False, bias=False, unconstrained=True)


def test_stalled_kernel_times_out_reports_and_recovers():
    w, t = _case()
    td = to_dev(t)
    assert kernel_name(w, td) == "tcgen05_bf16"
    assert dcn.dcn1d_device_status() == 0          # nothing pending from earlier tests
    out = torch.full((w.B, w.C_out, w.L_out), 7.0, dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    st = B.dcn1d_test_forward_stalled(td["x"], td["offsets"], td["weight"], w.stride,
                                      w.padding, w.dilation, w.groups, w.offset_groups,
                                      w.unconstrained, out=out, wait_limit_ns=1_000_000)
    assert st == 0, dcn.dcn1d_status_string(st)
    assert dcn.dcn1d_device_status() == DCN1D_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 10.0          # the call came back on its own
    assert bool((out == 7.0).all())                 # the stalled kernel stored nothing
    assert dcn.dcn1d_device_status() == 0           # the word was cleared by the read
    # the context is intact: an ordinary forward is correct and clean
    y = gpu_forward(w, td)
    assert dcn.dcn1d_device_status() == 0
    assert norm_err(y.double().cpu().numpy(), oracle_full(w, t)) <= TOL["bf16"]


def test_stalled_hook_rejects_other_shapes_and_limits():
    w, t = _case()
    td = to_dev(t)
    a = (td["x"], td["offsets"], td["weight"], w.stride, w.padding, w.dilation, w.groups,
         w.offset_groups, w.unconstrained)
    assert B.dcn1d_test_forward_stalled(*a, wait_limit_ns=10) == 4          # DCN1D_ERR_ARG
    assert B.dcn1d_test_forward_stalled(*a, wait_limit_ns=10**9) == 4
    w5, t5 = W.small_case(3, B=1, C_in=64, C_out=64, K=5, stride=1, padding=2, dilation=1,
                          groups=1, offset_groups=1, L_in=256, L_out=256, dtype="bf16")
    t5 = to_dev(t5)
    st = B.dcn1d_test_forward_stalled(t5["x"], t5["offsets"], t5["weight"], 1, 2, 1, 1, 1,
                                      False)
    assert st == 5                                                            # UNSUPPORTED
    assert dcn.dcn1d_device_status() == 0
