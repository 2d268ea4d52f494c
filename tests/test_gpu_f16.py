"""float16 inputs (the dc1d page's demo notebook: sampling positions survive float16) on
every path that takes them, against the oracle (GPU).

Tolerance: max|y - r| / max|r| <= 5e-3.  Outputs are rounded to fp16 (2^-11 relative);
the tensor-core path also interpolates in half2 arithmetic, so each sampled operand carries
a few fp16 roundings before the fp32 accumulation."""
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import TOL, gpu_forward, kernel_name, norm_err, oracle_full, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, off_scale, kernel
    ("tc_k5_mask_og4", 2, 128, 128, 5, 256, 1, 2, 1, 1, 4, True, False, 3.0, "tcgen05_f16"),
    ("tc_k9_strided_groups2_unc", 2, 256, 128, 9, 264, 2, 4, 2, 2, 2, False, True, 2.0,
     "tcgen05_f16"),
    ("tc_far_offsets_slow_taps", 2, 64, 64, 5, 256, 1, 2, 1, 1, 1, False, True, 80.0,
     "tcgen05_f16"),
    ("direct_ragged", 3, 6, 10, 3, 77, 2, 1, 2, 2, 3, True, False, 2.0, "direct"),
    ("depthwise_shape_takes_direct", 2, 32, 32, 3, 400, 1, 8, 8, 32, 32, False, True, 4.0,
     "direct"),
]


def _case(case, seed=17):
    name, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, sc, kern = case
    L_out = oracle.out_length(L, K, s, p, d)
    return W.small_case(seed, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype="f16",
                        mask=mask, unconstrained=unc, off_scale=sc)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_f16_forward_matches_oracle(case):
    w, t = _case(case)
    assert t["x"].dtype == torch.float16
    td = to_dev(t)
    assert kernel_name(w, td) == case[-1]
    y = gpu_forward(w, td)
    assert y.dtype == torch.float16
    assert dcn.dcn1d_device_status() == 0
    err = norm_err(y.double().cpu().numpy(), oracle_full(w, t))
    assert err <= TOL["f16"], (case[0], err)


def test_f16_sample_index_bit_exact():
    """Integer neighbours and fractions from fp16 offsets match the oracle bit for bit."""
    w, t = _case(CASES[1])
    offs = t["offsets"]
    i0, fr = dcn.dcn1d_sample_index(offs.cuda(), w.L_in, w.stride, w.padding, w.dilation,
                                    w.unconstrained)
    ri0, rfr = oracle.sample_index(offs, w.L_in, w.K, w.stride, w.padding, w.dilation,
                                   w.unconstrained)
    assert torch.equal(i0.cpu(), torch.from_numpy(ri0))
    assert torch.equal(fr.cpu().view(torch.int32), torch.from_numpy(rfr).view(torch.int32))


def test_f16_backward_matches_oracle():
    w, t = _case(CASES[0])
    td = to_dev(t)
    gout = torch.randn(w.B, w.C_out, w.L_out,
                       generator=torch.Generator().manual_seed(3)).to(torch.float16)
    got = dcn.dcn1d_backward(td["x"], td["offsets"], td["mask"], td["weight"], gout.cuda(),
                             w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                             w.unconstrained)
    torch.cuda.synchronize()
    ref = oracle.backward(t["x"], t["offsets"], t["mask"], t["weight"], gout, w.stride,
                          w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    for n, g in got.items():
        assert g.dtype == torch.float16
        err = norm_err(g.double().cpu().numpy(), ref["grad_" + n])
        assert err <= TOL["f16"], (n, err)
