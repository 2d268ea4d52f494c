"""Padding given per side, "valid" and "same" (the dc1d page's padding strings), on every
kernel family and in the backward, against the oracle (GPU)."""
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import TOL, norm_err, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, C_in, C_out, K, L_in, s, padding, d, groups, og, mask, unc, kernel
    ("direct_f32_same_odd_span", "f32", 2, 6, 4, 4, 37, 1, "same", 1, 2, 3, True, False,
     "direct"),
    ("direct_f32_pair_strided", "f32", 2, 4, 8, 3, 41, 2, (0, 3), 2, 1, 2, False, True,
     "direct"),
    ("depthwise_bf16_same", "bf16", 2, 32, 32, 4, 500, 1, "same", 3, 32, 32, False, True,
     "depthwise"),
    ("tc_bf16_same_k4", "bf16", 2, 128, 128, 4, 512, 1, "same", 1, 1, 4, True, False,
     "tcgen05_bf16"),
    ("tc_bf16_pair", "bf16", 1, 128, 64, 9, 264, 1, (5, 1), 1, 1, 1, False, True,
     "tcgen05_bf16"),
    ("tc_tf32_same_k16_d3", "f32", 2, 64, 64, 16, 128, 1, "same", 3, 1, 1, False, False,
     "tcgen05_3xtf32"),
]


def _setup(case, seed=9):
    name, dt, B, Ci, Co, K, L, s, pad, d, G, og, mask, unc, kern = case
    pl, pr = dcn.resolve_padding(pad, K, s, d)
    L_out = oracle.out_length(L, K, s, (pl, pr), d)
    w, t = W.small_case(seed, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=pl, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype=dt, mask=mask,
                        unconstrained=unc, off_scale=2.5)
    return w, t, pad, (pl, pr)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_forward_with_padding_per_side(case):
    w, t, pad, pads = _setup(case)
    td = to_dev(t)
    if pad == "same":
        assert w.L_out == w.L_in
    assert dcn.dcn1d_forward_kernel_name(td["x"], td["offsets"], td["mask"], td["weight"],
                                         td["bias"], w.stride, pad, w.dilation, w.groups,
                                         w.offset_groups, w.unconstrained) == case[-1]
    y = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"], w.stride,
                          pad, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    r = oracle.forward(t["x"], t["offsets"], t["mask"], t["weight"], t["bias"], w.stride, pads,
                       w.dilation, w.groups, w.offset_groups, w.unconstrained)
    assert y.shape == tuple(r.shape)
    err = norm_err(y.double().cpu().numpy(), r)
    assert err <= TOL[w.dtype], (case[0], err)


@pytest.mark.parametrize("case", [CASES[0], CASES[3]], ids=[CASES[0][0], CASES[3][0]])
def test_backward_with_padding_per_side(case):
    w, t, pad, pads = _setup(case)
    td = to_dev(t)
    gout = torch.randn(w.B, w.C_out, w.L_out,
                       generator=torch.Generator().manual_seed(5)).to(t["x"].dtype)
    got = dcn.dcn1d_backward(td["x"], td["offsets"], td["mask"], td["weight"], gout.cuda(),
                             w.stride, pad, w.dilation, w.groups, w.offset_groups,
                             w.unconstrained)
    torch.cuda.synchronize()
    ref = oracle.backward(t["x"], t["offsets"], t["mask"], t["weight"], gout, w.stride, pads,
                          w.dilation, w.groups, w.offset_groups, w.unconstrained)
    for n, g in got.items():
        err = norm_err(g.double().cpu().numpy(), ref["grad_" + n])
        assert err <= TOL[w.dtype], (case[0], n, err)


def test_symmetric_pair_equals_int_padding():
    case = ("pair_vs_int", "f32", 2, 4, 8, 3, 41, 2, 2, 2, 1, 2, False, True, "direct")
    w, t, _, _ = _setup(case)
    td = to_dev(t)
    args = (td["x"], td["offsets"], td["mask"], td["weight"], td["bias"], w.stride)
    rest = (w.dilation, w.groups, w.offset_groups, w.unconstrained)
    a = dcn.dcn1d_forward(*args, 2, *rest)
    b = dcn.dcn1d_forward(*args, (2, 2), *rest)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_padding_errors():
    case = CASES[1]
    w, t, _, _ = _setup(case)
    td = to_dev(t)
    with pytest.raises(ValueError):   # "same" with stride 2
        dcn.dcn1d_forward(td["x"], td["offsets"], None, td["weight"], None, 2, "same",
                          w.dilation, w.groups, w.offset_groups, w.unconstrained)
    with pytest.raises(dcn.Dcn1dError) as e:   # negative right padding
        dcn.dcn1d_forward(td["x"], td["offsets"], None, td["weight"], None, w.stride, (0, -1),
                          w.dilation, w.groups, w.offset_groups, w.unconstrained)
    assert e.value.status == 4
