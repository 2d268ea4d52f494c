"""PackedDeformConv1d (the dc1d page's "PackedDeformConv1d" and "Modulation (DCNv2)"):
the offset and mask trunk and the whole layer through the C ABI, against the oracle (GPU).

Tolerances (normwise, max|y - r| / max|r|, per tensor): the TOL of the dtype.  The trunk
keeps its depthwise output in fp32 on chip; the tensor-core kernel rounds it once to the
16-bit input type before the pointwise contraction (fp32 accumulation), one rounding more
than the layer's tensors themselves carry.  The layer's output is compared with the oracle
layer, whose predicted offsets and mask are rounded to the layer's dtype before its forward,
as the layer passes them on.
"""
import numpy as np
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import TOL, norm_err

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, C_in, C_out, K, L_in, stride, padding, dilation, groups, og, modulated,
    # biases, trunk kernel
    ("page_example_bf16", "bf16", 2, 64, 64, 3, 300, 1, "same", 4, 64, 64, True, True,
     "trunk_tcgen05"),
    ("og8_k5_ragged_bf16", "bf16", 2, 128, 128, 5, 257, 1, (2, 2), 1, 1, 8, True, True,
     "trunk_tcgen05"),
    ("strided_asym_nobias_f16", "f16", 1, 192, 64, 4, 203, 2, (1, 2), 1, 1, 3, False, False,
     "trunk_tcgen05"),
    ("two_chunks_per_head_bf16", "bf16", 1, 512, 128, 3, 200, 1, (1, 1), 1, 4, 128, True, True,
     "trunk_tcgen05"),
    ("k9_single_group_f16", "f16", 1, 64, 32, 9, 150, 1, (4, 4), 1, 1, 1, True, True,
     "trunk_tcgen05"),
    ("simt_f32", "f32", 2, 6, 4, 3, 41, 1, "same", 2, 2, 3, True, True, "trunk_simt"),
    ("simt_bf16_cin48", "bf16", 2, 48, 48, 3, 77, 2, (3, 0), 1, 48, 48, True, True,
     "trunk_simt"),
]
IDS = [c[0] for c in CASES]


def setup(case, seed=11):
    (name, dt, B, Ci, Co, K, L, s, pad, d, G, og, modulated, biases, kern) = case
    pl, pr = dcn.resolve_padding(pad, K, s, d)
    L_out = oracle.out_length(L, K, s, (pl, pr), d)
    w, t = W.packed_case(seed, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=pl, dilation=d,
                         groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype=dt,
                         modulated=modulated, biases=biases)
    return w, t, pad, (pl, pr)


def dev(t):
    return {k: (v.cuda() if v is not None else None) for k, v in t.items()}


TRUNK_KEYS = ("x", "dw_weight", "dw_bias", "off_weight", "off_bias", "mask_weight", "mask_bias")


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_trunk_matches_oracle(case):
    w, t, pad, pads = setup(case)
    td = dev(t)
    args = [td[k] for k in TRUNK_KEYS]
    assert dcn.dcn1d_packed_trunk_kernel_name(*args, w.stride, pad, w.dilation,
                                              w.offset_groups) == case[-1]
    off, mask = dcn.dcn1d_packed_trunk(*args, w.stride, pad, w.dilation, w.offset_groups)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    roff, rmask = oracle.packed_trunk(*[t[k] for k in TRUNK_KEYS], w.K, w.stride, pads,
                                      w.dilation, w.offset_groups)
    assert off.dtype == t["x"].dtype and tuple(off.shape) == roff.shape
    assert norm_err(off.double().cpu().numpy(), roff) <= TOL[w.dtype]
    assert (mask is None) == (rmask is None)
    if mask is not None:
        assert norm_err(mask.double().cpu().numpy(), rmask) <= TOL[w.dtype]


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_packed_layer_matches_oracle(case):
    w, t, pad, pads = setup(case)
    td = dev(t)
    y, extra = dcn.dcn1d_packed_forward(*[td[k] for k in TRUNK_KEYS], td["weight"], td["bias"],
                                        w.stride, pad, w.dilation, w.groups, w.offset_groups,
                                        False, with_offsets=True)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    ry, roff, rmask = oracle.packed_forward(*[t[k] for k in TRUNK_KEYS], t["weight"], t["bias"],
                                            w.stride, pads, w.dilation, w.groups,
                                            w.offset_groups, False)
    assert tuple(y.shape) == ry.shape
    assert norm_err(y.double().cpu().numpy(), ry) <= TOL[w.dtype], case[0]
    off, mask = extra if rmask is not None else (extra, None)
    assert norm_err(off.double().cpu().numpy(), roff) <= TOL[w.dtype]
    if rmask is not None:
        assert norm_err(mask.double().cpu().numpy(), rmask) <= TOL[w.dtype]
    # without with_offsets the predicted tensors stay in the workspace; same output
    y2 = dcn.dcn1d_packed_forward(*[td[k] for k in TRUNK_KEYS], td["weight"], td["bias"],
                                  w.stride, pad, w.dilation, w.groups, w.offset_groups, False)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_zero_initialised_mask_head_gives_half():
    """The page: the mask head's final projection starts at zero, so every tap's mask is
    exactly 0.5 and the output (less its bias) is half the unmodulated layer's."""
    case = CASES[0]
    w, t, pad, pads = setup(case)
    t["mask_weight"] = torch.zeros_like(t["mask_weight"])
    t["mask_bias"] = torch.zeros_like(t["mask_bias"])
    td = dev(t)
    rest = (td["weight"], td["bias"], w.stride, pad, w.dilation, w.groups, w.offset_groups,
            False)
    y_mod, (off, mask) = dcn.dcn1d_packed_forward(*[td[k] for k in TRUNK_KEYS], *rest,
                                                  with_offsets=True)
    y_plain = dcn.dcn1d_packed_forward(td["x"], td["dw_weight"], td["dw_bias"],
                                       td["off_weight"], td["off_bias"], None, None, *rest)
    torch.cuda.synchronize()
    assert torch.all(mask == 0.5)
    b = td["bias"].float()[None, :, None]
    lhs, rhs = (y_mod.float() - b), 0.5 * (y_plain.float() - b)
    assert norm_err(lhs.double().cpu().numpy(), rhs.double().cpu().numpy()) <= TOL[w.dtype]


def test_packed_errors_and_empty_batch():
    w, t, pad, pads = setup(CASES[5])
    td = dev(t)
    args = [td[k] for k in TRUNK_KEYS]
    off, mask = dcn.dcn1d_packed_trunk(*args, w.stride, pad, w.dilation, w.offset_groups)
    with pytest.raises(dcn.Dcn1dError) as e:   # a mask output without a mask head
        dcn.dcn1d_packed_trunk(td["x"], td["dw_weight"], td["dw_bias"], td["off_weight"],
                               td["off_bias"], None, None, w.stride, pad, w.dilation,
                               w.offset_groups, offsets_out=off, mask_out=mask)
    assert e.value.status == 4
    with pytest.raises(dcn.Dcn1dError) as e:   # offset head of the wrong width
        dcn.dcn1d_packed_trunk(td["x"], td["dw_weight"], td["dw_bias"], td["off_weight"][:-1],
                               None, None, None, w.stride, pad, w.dilation, w.offset_groups)
    assert e.value.status == 3
    with pytest.raises(ValueError):            # workspace too small for the predicted tensors
        dcn.dcn1d_packed_forward(*args, td["weight"], td["bias"], w.stride, pad, w.dilation,
                                 w.groups, w.offset_groups, False,
                                 workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    empty = {k: (v[:0] if k == "x" else v) for k, v in td.items()}
    y = dcn.dcn1d_packed_forward(*[empty[k] for k in TRUNK_KEYS], td["weight"], td["bias"],
                                 w.stride, pad, w.dilation, w.groups, w.offset_groups, False)
    assert y.shape[0] == 0 and dcn.dcn1d_last_launch_count() == 0


def test_packed_workload_sampled_against_oracle():
    """The packed workload at full size, in the bench's launch configuration: the trunk's
    outputs and the layer's output on sampled positions against the oracle."""
    w = W.PACKED_MODULATED_BF16
    t = W.make_packed_inputs(w, seed=0)
    td = dev(t)
    y, (off, mask) = dcn.dcn1d_packed_forward(*[td[k] for k in TRUNK_KEYS], td["weight"],
                                              td["bias"], w.stride, w.padding, w.dilation,
                                              w.groups, w.offset_groups, False,
                                              with_offsets=True)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    # the trunk on a window of positions: run the oracle on a slice of the signal that
    # holds every tap of output positions [l0, l0 + n)
    rng = np.random.default_rng(0)
    span = w.dilation * (w.K - 1)
    for b in (0, w.B - 1):
        for l0 in rng.integers(0, w.L_out - 64, size=2):
            lo = max(0, l0 - w.padding)
            hi = min(w.L_in, l0 + 64 - w.padding + span)
            sl = {k: v for k, v in t.items()}
            sl["x"] = t["x"][b:b + 1, :, lo:hi]
            pl = max(0, w.padding - l0)
            pr = max(0, (l0 + 64 - w.padding + span) - w.L_in)
            roff, rmask = oracle.packed_trunk(*[sl[k] for k in TRUNK_KEYS], w.K, w.stride,
                                              (pl, pr), w.dilation, w.offset_groups)
            got_off = off[b:b + 1, :, l0:l0 + 64].double().cpu().numpy()
            got_mask = mask[b:b + 1, :, l0:l0 + 64].double().cpu().numpy()
            assert norm_err(got_off, roff) <= TOL["bf16"]
            assert norm_err(got_mask, rmask) <= TOL["bf16"]
    # the layer's output at sampled points, from the kernel's own predicted tensors
    pts = np.stack([rng.integers(0, w.B, 2000), rng.integers(0, w.C_out, 2000),
                    rng.integers(0, w.L_out, 2000)], axis=1)
    r = oracle.forward_points(t["x"], off.cpu(), mask.cpu(), t["weight"], t["bias"], w.stride,
                              w.padding, w.dilation, w.groups, w.offset_groups, False, pts)
    yv = y.cpu()[pts[:, 0], pts[:, 1], pts[:, 2]].double().numpy()
    assert norm_err(yv, r) <= TOL["bf16"]
