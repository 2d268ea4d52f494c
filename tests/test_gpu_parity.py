"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs.  Integer decisions (floor positions, clamps) must match bit for bit; outputs within
the normwise bound max|y - r| / max|r| <= 1e-4 (fp32) or 2e-2 (bf16 inputs, fp32
accumulation)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import (TOL, gpu_forward, inputs, kernel_name, norm_err, oracle_full,
                      oracle_points, reduced, sample_points, to_dev)

pytestmark = pytest.mark.gpu

# Reduced sizes of the five workloads: the oracle finishes them in seconds, and each still
# spans several tiles of every kernel with a ragged tail.
REDUCED = [
    reduced(W.TINY_F32),
    reduced(W.USAGE_F32, B=2),
    reduced(W.DEPTHWISE_BF16, B=2, C_in=64, C_out=64, groups=64, offset_groups=64, L_in=3001),
    reduced(W.MODULATED_BF16, B=2, L_in=336),   # L_out 336 = 2 tiles of 128 + 80
    reduced(W.LARGE_BF16, B=2, L_in=696),       # L_out 344 = 2 tiles of 128 + 88
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dcn.load()


@pytest.mark.parametrize("w", REDUCED, ids=[w.name for w in REDUCED])
def test_reduced_workload_full_parity(w):
    t = W.make_inputs(w, seed=1)
    td = to_dev(t)
    y = gpu_forward(w, td)
    torch.cuda.synchronize()
    r = oracle_full(w, t)
    err = norm_err(y.double().cpu().numpy(), r)
    assert err <= TOL[w.dtype], (w.name, kernel_name(w, td), err)


@pytest.mark.parametrize("w", W.ORDERED, ids=[w.name for w in W.ORDERED])
def test_full_size_sampled_parity(w):
    """Full workload size, the same entry point and kernel the bench times; outputs sampled."""
    t = inputs(w, 0)
    td = to_dev(t)
    y = gpu_forward(w, td)
    torch.cuda.synchronize()
    rows = [(0, 0), (w.B - 1, w.C_out - 1), (w.B // 2, w.C_out // 3)]
    pts = sample_points(w, 4096, seed=7, rows=rows)
    r = oracle_points(w, t, pts)
    yc = y.double().cpu().numpy()[pts[:, 0], pts[:, 1], pts[:, 2]]
    err = norm_err(yc, r)
    assert err <= TOL[w.dtype], (w.name, kernel_name(w, td), err)
    assert torch.isfinite(y).all()


@pytest.mark.parametrize("w", W.ORDERED, ids=[w.name for w in W.ORDERED])
def test_sample_index_bit_exact(w):
    """floor positions and fractions of every tap (first batch element for the big ones)."""
    t = inputs(w, 0)
    offs = t["offsets"][:1] if t["offsets"].numel() > 4_000_000 else t["offsets"]
    i0, fr = dcn.dcn1d_sample_index(offs.cuda(), w.L_in, w.stride, w.padding, w.dilation,
                                    w.unconstrained)
    ri0, rfr = oracle.sample_index(offs, w.L_in, w.K, w.stride, w.padding, w.dilation,
                                   w.unconstrained)
    assert np.array_equal(i0.cpu().numpy(), ri0)
    assert np.array_equal(fr.cpu().numpy().view(np.int32), rfr.view(np.int32))


EDGE = [
    # name, B, C_in, C_out, K, L_in, s, p, d, groups, og, dtype, mask, unc, off_scale
    ("k1", 2, 8, 8, 1, 37, 1, 0, 1, 1, 1, "f32", False, False, 3.0),
    ("k1_unc", 2, 8, 8, 1, 37, 1, 0, 1, 1, 2, "bf16", True, True, 3.0),
    ("stride3", 2, 16, 24, 4, 70, 3, 2, 2, 2, 4, "f32", True, False, 2.0),
    ("pad_past_span", 1, 8, 16, 3, 9, 1, 7, 1, 1, 1, "f32", False, True, 2.0),
    ("far_offsets", 2, 8, 8, 3, 40, 1, 1, 1, 1, 8, "bf16", False, True, 60.0),
    ("lout1", 3, 8, 12, 5, 5, 1, 0, 1, 1, 1, "f32", True, False, 1.0),
    ("lout1_stride", 2, 4, 4, 3, 6, 5, 0, 2, 2, 2, "bf16", False, True, 1.0),
    ("cout_ragged", 2, 32, 200, 3, 65, 1, 1, 1, 1, 4, "bf16", False, False, 2.0),
    ("og_ne_groups", 2, 24, 16, 3, 50, 2, 1, 3, 4, 3, "f32", True, True, 4.0),
    ("depthwise_small", 2, 32, 32, 3, 300, 1, 8, 8, 32, 32, "bf16", False, True, 4.0),
    ("depthwise_constrained", 2, 16, 16, 5, 129, 2, 4, 2, 16, 16, "f32", True, False, 3.0),
    ("grouped_dw_mult", 1, 8, 16, 3, 40, 1, 1, 1, 8, 8, "f32", False, False, 2.0),
    ("dense_bf16_mid", 2, 128, 256, 5, 300, 1, 2, 1, 1, 8, "bf16", True, False, 3.0),
    ("dense_bf16_strided", 1, 256, 128, 9, 257, 2, 4, 2, 2, 2, "bf16", False, True, 2.0),
    ("dense_f32_mid", 2, 64, 96, 7, 120, 1, 3, 2, 1, 2, "f32", False, False, 1.5),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_cases(case):
    name, B, Ci, Co, K, L, s, p, d, G, og, dt, mask, unc, sc = case
    L_out = oracle.out_length(L, K, s, p, d)
    assert L_out >= 1
    w, t = W.small_case(11, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype=dt, mask=mask,
                        unconstrained=unc, off_scale=sc)
    td = to_dev(t)
    y = gpu_forward(w, td)
    torch.cuda.synchronize()
    r = oracle_full(w, t)
    err = norm_err(y.double().cpu().numpy(), r)
    assert err <= TOL[dt], (name, kernel_name(w, td), err)


def test_integer_and_exact_positions():
    """Offsets that land exactly on integers, on the receptive-field edges and on .5."""
    w, t = W.small_case(12, B=2, C_in=16, C_out=16, K=3, stride=2, padding=2, dilation=2,
                        groups=1, offset_groups=4, L_in=64, L_out=oracle.out_length(64, 3, 2, 2, 2),
                        dtype="f32", mask=False, unconstrained=False)
    g = torch.Generator().manual_seed(5)
    t["offsets"] = (torch.randint(-8, 9, t["offsets"].shape, generator=g) * 0.5).float()
    td = to_dev(t)
    for unc in (False, True):
        y = gpu_forward(w, td, unconstrained=unc)
        r = oracle.forward(t["x"], t["offsets"], None, t["weight"], t["bias"], w.stride,
                           w.padding, w.dilation, w.groups, w.offset_groups, unc)
        assert norm_err(y.double().cpu().numpy(), r) <= 1e-5


@pytest.mark.parametrize("w", [W.USAGE_F32, W.MODULATED_BF16, W.LARGE_BF16, W.DEPTHWISE_BF16],
                         ids=lambda w: w.name)
def test_mask_ones_bitwise_equals_no_mask(w):
    """dc1d "Modulation (DCNv2)": an all-ones mask gives bit-for-bit the no-mask output."""
    w2 = w.with_batch(min(w.B, 2))
    t = W.make_inputs(w2, seed=3)
    td = to_dev(t)
    a = gpu_forward(w2, td, mask=None)
    b = gpu_forward(w2, td, mask=torch.ones_like(td["offsets"]))
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16 if a.dtype == torch.bfloat16 else torch.int32),
                       b.view(torch.int16 if b.dtype == torch.bfloat16 else torch.int32))


@pytest.mark.parametrize("w", W.ORDERED, ids=[w.name for w in W.ORDERED])
def test_zero_offsets_match_cudnn_conv1d(w):
    """Zero offsets reproduce conv1d (dc1d "Going faster": the zero-offset invariant);
    checked at full size against torch's own conv1d on the GPU in float32."""
    t = inputs(w, 0)
    td = to_dev(t)
    td["offsets"] = torch.zeros_like(td["offsets"])
    y = gpu_forward(w, td, mask=None)
    prev = torch.backends.cudnn.allow_tf32
    torch.backends.cudnn.allow_tf32 = False   # the reference itself must be true fp32
    try:
        ref = F.conv1d(td["x"].float(), td["weight"].float(),
                       td["bias"].float() if td["bias"] is not None else None, stride=w.stride,
                       padding=w.padding, dilation=w.dilation, groups=w.groups)
        torch.cuda.synchronize()
    finally:
        torch.backends.cudnn.allow_tf32 = prev
    err = (y.float() - ref).abs().max().item() / ref.abs().max().item()
    assert err <= TOL[w.dtype], (w.name, err)


def test_two_calls_same_bits_and_stream_order():
    """Deterministic: two calls give identical bits; a side stream is honoured."""
    w = reduced(W.MODULATED_BF16, B=2, L_in=1000)
    td = to_dev(W.make_inputs(w, seed=9))
    a = gpu_forward(w, td)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"],
                              w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                              w.unconstrained, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_empty_batch():
    w = reduced(W.USAGE_F32, B=1)
    td = to_dev(W.make_inputs(w, seed=0))
    x = td["x"][:0].contiguous()
    off = td["offsets"][:0].contiguous()
    y = dcn.dcn1d_forward(x, off, None, td["weight"], td["bias"], w.stride, w.padding,
                          w.dilation, w.groups, w.offset_groups, w.unconstrained)
    assert y.shape == (0, w.C_out, w.L_out)
    assert dcn.dcn1d_last_launch_count() == 0


def test_invalid_arguments_raise_on_gpu():
    w = reduced(W.USAGE_F32, B=1)
    td = to_dev(W.make_inputs(w, seed=0))
    with pytest.raises(dcn.Dcn1dError) as e:
        dcn.dcn1d_forward(td["x"], td["offsets"][:, :, :-1].contiguous(), None, td["weight"],
                          td["bias"], w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                          w.unconstrained)
    assert e.value.status == 3
    with pytest.raises(dcn.Dcn1dError) as e:
        dcn.dcn1d_forward(td["x"], td["offsets"], None, td["weight"].bfloat16(), td["bias"],
                          w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                          w.unconstrained)
    assert e.value.status == 2
