"""Backward pass through the C ABI against the oracle's backward (GPU).

Each gradient is compared normwise, max|g - r| / max|r|, with the forward's bounds: 1e-4
for fp32 inputs (fp32 arithmetic, sums of up to C_out/groups or B*L_out terms) and 2e-2
for bf16 inputs (gradients rounded to bf16 on output).
"""
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import TOL, norm_err, to_dev

pytestmark = pytest.mark.gpu

NAMES = {"x": "grad_x", "offsets": "grad_offsets", "mask": "grad_mask", "weight": "grad_weight",
         "bias": "grad_bias"}

CASES = [
    # name, dtype, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, off_scale
    ("f32_g2_og2_mask", "f32", 2, 8, 12, 3, 40, 1, 1, 1, 2, 2, True, False, 2.0),
    ("f32_strided_dilated_unc", "f32", 3, 16, 32, 5, 130, 2, 4, 2, 4, 4, False, True, 3.0),
    ("f32_depthwise", "f32", 2, 16, 16, 3, 300, 1, 8, 8, 16, 16, False, True, 4.0),
    ("f32_lout_1", "f32", 2, 32, 8, 16, 16, 1, 0, 1, 1, 1, False, False, 2.0),
    ("bf16_modulated_like", "bf16", 2, 64, 64, 5, 260, 1, 2, 1, 1, 8, True, False, 3.0),
    ("bf16_groups4_unc", "bf16", 2, 64, 64, 9, 200, 2, 4, 2, 4, 4, False, True, 2.0),
    # fp32 on the tensor cores: groups, mask, unconstrained, L_out not a multiple of 4
    ("f32_tc_g2_mask_unc", "f32", 3, 32, 64, 7, 150, 1, 3, 2, 2, 4, True, True, 3.0),
    ("f32_tc_strided_ragged", "f32", 2, 48, 32, 4, 203, 2, 1, 1, 1, 2, False, False, 2.0),
]


def _inputs(case, seed=7):
    name, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, sc = case
    L_out = oracle.out_length(L, K, s, p, d)
    w, t = W.small_case(seed, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype=dt, mask=mask,
                        unconstrained=unc, off_scale=sc)
    g = torch.Generator().manual_seed(seed + 1)
    gout = torch.randn(B, Co, L_out, generator=g).to(t["x"].dtype)
    return w, t, gout


def _run(w, t, gout, wanted=dcn.GRADS):
    td = to_dev(t)
    got = dcn.dcn1d_backward(td["x"], td["offsets"], td["mask"], td["weight"], gout.cuda(),
                             w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                             w.unconstrained, wanted=wanted)
    torch.cuda.synchronize()
    return got


def _ref(w, t, gout):
    return oracle.backward(t["x"], t["offsets"], t["mask"], t["weight"], gout, w.stride,
                           w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(case):
    w, t, gout = _inputs(case)
    got = _run(w, t, gout)
    ref = _ref(w, t, gout)
    for n, g in got.items():
        r = ref[NAMES[n]]
        assert g.shape == tuple(r.shape), n
        err = norm_err(g.double().cpu().numpy(), r)
        assert err <= TOL[w.dtype], (case[0], n, err)


# three TF32 products reach about fp32 accuracy; one product would give ~1e-4 here
TF32_SPLIT_BOUND = 1e-5


def test_backward_usage_shape_fp32():
    """The usage shape (C_in = C_out = 512, K = 16, dilation 3) at batch 2: its two
    contractions on the tensor cores by three TF32 products (L_out = 83, so the columns
    and grad_out of the weight gradient go through rows padded to a multiple of 4)."""
    w = W.USAGE_F32.with_batch(2)
    t = W.make_inputs(w, seed=3)
    gout = torch.randn(w.B, w.C_out, w.L_out, generator=torch.Generator().manual_seed(4))
    td = to_dev(t)
    assert dcn.dcn1d_backward_kernel_name(td["x"], td["offsets"], td["mask"], td["weight"],
                                          gout.cuda(), w.stride, w.padding, w.dilation,
                                          w.groups, w.offset_groups,
                                          w.unconstrained) == "tcgen05_gemm"
    got = _run(w, t, gout)
    assert dcn.dcn1d_device_status() == 0
    ref = _ref(w, t, gout)
    for n, g in got.items():
        err = norm_err(g.double().cpu().numpy(), ref[NAMES[n]])
        assert err <= TF32_SPLIT_BOUND, (n, err)


# the CUDA-core fp32 path, the fp32 tensor-core path (padded rows), and the 16-bit path
# whose column-gradient GEMM drains into the sampling gradient
SUBSET_CASES = [CASES[0], CASES[7], CASES[4]]


@pytest.mark.parametrize("case", SUBSET_CASES, ids=[c[0] for c in SUBSET_CASES])
def test_backward_subsets_match_the_full_call(case):
    """Asking for fewer gradients gives the same values for those asked (grad_weight and
    grad_bias are summed in a fixed order: the same bits)."""
    w, t, gout = _inputs(case)
    full = _run(w, t, gout)
    part = _run(w, t, gout, wanted=("weight", "bias"))
    assert set(part) == {"weight", "bias"}
    assert torch.equal(part["weight"], full["weight"])
    assert torch.equal(part["bias"], full["bias"])
    # grad_x and grad_offsets are fp32 atomic sums (their order varies), rounded once to
    # the dtype: a bf16 result may move by one unit in its last place
    tol = 1e-6 if w.dtype == "f32" else 1e-2
    only_x = _run(w, t, gout, wanted=("x",))
    assert norm_err(only_x["x"].double().cpu().numpy(),
                    full["x"].double().cpu().numpy()) <= tol
    only_off = _run(w, t, gout, wanted=("offsets",))
    assert norm_err(only_off["offsets"].double().cpu().numpy(),
                    full["offsets"].double().cpu().numpy()) <= tol


def test_backward_clamped_offsets_get_zero_gradient():
    """Constrained mode with every tap pushed far outside its receptive field."""
    case = CASES[0]
    w, t, gout = _inputs(case)
    t["offsets"] = torch.where(torch.arange(t["offsets"].numel()).view_as(t["offsets"]) % 2 == 0,
                               torch.tensor(60.5), torch.tensor(-60.5))
    got = _run(w, t, gout, wanted=("offsets",))
    assert torch.count_nonzero(got["offsets"]) == 0


def test_backward_empty_batch():
    case = CASES[0]
    w, t, gout = _inputs(case)
    w0 = w.with_batch(0)
    t0 = {k: (v[:0] if (v is not None and k in ("x", "offsets", "mask")) else v)
          for k, v in t.items()}
    got = _run(w0, t0, gout[:0])
    assert got["x"].numel() == 0 and got["offsets"].numel() == 0
    assert torch.count_nonzero(got["weight"]) == 0
    assert torch.count_nonzero(got["bias"]) == 0


def test_backward_rejects_bad_arguments():
    case = CASES[1]   # no mask
    w, t, gout = _inputs(case)
    td = to_dev(t)
    bad_mask_grad = {"mask": torch.empty_like(td["offsets"])}
    with pytest.raises(dcn.Dcn1dError) as e:
        dcn.dcn1d_backward(td["x"], td["offsets"], None, td["weight"], gout.cuda(), w.stride,
                           w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained,
                           wanted=("x",), grads=bad_mask_grad)
    assert e.value.status == 4   # DCN1D_ERR_ARG: a mask gradient without a mask
    with pytest.raises(dcn.Dcn1dError) as e:
        dcn.dcn1d_backward(td["x"], td["offsets"], None, td["weight"], gout[:, :1].cuda(),
                           w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                           w.unconstrained)
    assert e.value.status == 3   # DCN1D_ERR_SHAPE: grad_out is not [B, C_out, L_out]
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        dcn.dcn1d_backward(td["x"], td["offsets"], None, td["weight"], gout.cuda(), w.stride,
                           w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained,
                           workspace=ws[:16])
