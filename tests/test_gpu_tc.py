"""GPU parity of the fused tensor-core (tcgen05) bf16 path: shapes chosen so that the
library selects it, asserted, then compared with the oracle; plus the device status word
(no bounded wait may have given up)."""
import numpy as np
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import (TOL, gpu_forward, kernel_name, norm_err, oracle_full, oracle_points,
                      sample_points, to_dev)

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, off_scale
    ("g1_k5_mask_constrained", 2, 128, 128, 5, 256, 1, 2, 1, 1, 4, True, False, 3.0),
    ("g2_k9_strided_unc", 2, 256, 128, 9, 264, 2, 4, 2, 2, 2, False, True, 2.0),
    ("g4_k4_cout32", 1, 128, 128, 4, 512, 1, 1, 1, 4, 4, False, True, 4.0),
    ("g1_k4_cout96_ragged", 3, 64, 96, 4, 200, 1, 3, 3, 1, 1, True, True, 2.0),
    ("g1_k7_og_per_32", 1, 64, 64, 7, 136, 1, 3, 1, 1, 2, False, False, 2.5),
    ("far_offsets_slow_taps", 2, 64, 64, 5, 256, 1, 2, 1, 1, 1, False, True, 80.0),
    ("l_out_below_one_tile", 2, 128, 256, 5, 64, 1, 2, 1, 1, 4, True, False, 3.0),
    # more than 256 output channels per conv group: blocks of 256, and of 192
    ("cout_512_two_blocks", 2, 128, 512, 5, 256, 1, 2, 1, 1, 4, True, False, 3.0),
    ("g2_cout_g384_blocks_of_192", 1, 128, 768, 3, 200, 1, 1, 1, 2, 2, False, True, 2.0),
    # the dc1d page's usage layer (kernel 16, dilation 3) in bf16: narrower, then its own
    # 512 channels; tap positions of wide kernels live in shared memory
    ("k16_d3_usage_like", 2, 128, 128, 16, 128, 1, 0, 3, 1, 1, False, False, 1.5),
    ("k16_d3_usage_channels", 1, 512, 512, 16, 128, 1, 0, 3, 1, 1, False, False, 1.5),
    ("k16_mask_og2_unc_far", 2, 64, 64, 16, 200, 1, 8, 2, 1, 2, True, True, 40.0),
    # L_in not a multiple of 8: x windows by the loader's 4-byte copies (one box, two
    # boxes, taps past the window)
    ("lin300_copy_k5_mask", 2, 128, 128, 5, 300, 1, 2, 1, 1, 4, True, False, 3.0),
    ("lin330_copy_k9_strided_two_boxes", 2, 128, 128, 9, 330, 2, 4, 2, 2, 2, False, True, 2.0),
    ("lin202_copy_far_offsets", 3, 64, 64, 3, 202, 1, 1, 1, 1, 1, False, True, 80.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_bf16_parity(case):
    name, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, sc = case
    L_out = oracle.out_length(L, K, s, p, d)
    w, t = W.small_case(21, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype="bf16",
                        mask=mask, unconstrained=unc, off_scale=sc)
    td = to_dev(t)
    assert kernel_name(w, td) == "tcgen05_bf16", kernel_name(w, td)
    y = gpu_forward(w, td)
    assert dcn.dcn1d_device_status() == 0
    r = oracle_full(w, t)
    err = norm_err(y.double().cpu().numpy(), r)
    assert err <= TOL["bf16"], (name, err)


@pytest.mark.parametrize("w", [W.MODULATED_BF16, W.LARGE_BF16], ids=lambda w: w.name)
def test_named_dense_workloads_take_the_tensor_core_path(w):
    t = W.make_inputs(w.with_batch(1), seed=0)
    td = to_dev(t)
    assert kernel_name(w.with_batch(1), td) == "tcgen05_bf16"


# Several tiles a CTA (more than 3 x 148), so the accumulator's placement cycles: channel
# blocks of 128 rotate over three 128-column slots; wider ones alternate between columns
# [0, N) and [128, 128 + N), sharing [128, 256) with the next tile.  The last case leaves
# no room for the drain's parked values (16 KB of bias), so the shared slot is stored
# before its release.
MANY_TILES = [
    # name, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, off_scale
    ("n128_three_slots", 8, 32, 128, 4, 10240, 1, 1, 1, 1, 2, True, False, 2.0),
    ("n256_alternating_parked", 8, 32, 256, 4, 10240, 1, 2, 1, 1, 1, False, True, 3.0),
    ("n192_alternating_parked", 6, 64, 192, 4, 12288, 1, 1, 1, 1, 4, True, True, 2.0),
    ("n256_alternating_no_room_to_park", 1, 1024, 4096, 9, 8192, 2, 4, 2, 16, 16, False,
     True, 2.0),
    # last rounds of 50 and 60 tiles, split between the CTAs of 2-CTA clusters: three
    # k-blocks (halves of one and two), and K = 16 in two 256-channel blocks
    ("k3_mask_odd_kblocks_split_tail", 6, 64, 256, 3, 13696, 1, 1, 1, 1, 2, True, False, 2.0),
    ("k16_two_blocks_split_tail", 2, 128, 512, 16, 16048, 1, 0, 3, 1, 1, False, False, 1.5),
]


@pytest.mark.parametrize("case", MANY_TILES, ids=[c[0] for c in MANY_TILES])
def test_tc_bf16_many_tiles_per_cta(case):
    name, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, sc = case
    L_out = oracle.out_length(L, K, s, p, d)
    w, t = W.small_case(23, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype="bf16",
                        mask=mask, unconstrained=unc, off_scale=sc)
    td = to_dev(t)
    assert kernel_name(w, td) == "tcgen05_bf16", kernel_name(w, td)
    y = gpu_forward(w, td)
    assert dcn.dcn1d_device_status() == 0
    # every channel of two positions in each of several tiles, both halves of the
    # channel block, plus whole rows and random points
    ls = sorted({0, 127, 128, 255, 256 + 77, 3 * 128 + 5, L_out // 2, L_out - 1})
    bs = sorted({0, B - 1})
    grid = np.array([(b, co, l) for b in bs for l in ls for co in range(Co)], dtype=np.int64)
    rows = [(0, 0), (B - 1, Co - 1), (0, 128 % Co), (B - 1, Co // 2 - 1)]
    pts = np.concatenate([grid, sample_points(w, 4096, seed=11, rows=rows)])
    r = oracle_points(w, t, pts)
    yc = y.double().cpu().numpy()[pts[:, 0], pts[:, 1], pts[:, 2]]
    err = norm_err(yc, r)
    assert err <= TOL["bf16"], (name, err)


def test_device_status_clean_after_many_launches():
    w, t = W.small_case(5, B=2, C_in=128, C_out=128, K=5, stride=1, padding=2, dilation=1,
                        groups=1, offset_groups=4, L_in=512, L_out=512, dtype="bf16")
    td = to_dev(t)
    ys = [gpu_forward(w, td) for _ in range(20)]
    assert dcn.dcn1d_device_status() == 0
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))


# ---------------------------------------------------------------- fp32: 3xTF32 tensor-core path

TF32_CASES = [
    # name, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, off_scale
    ("usage_shape_b2_split", 2, 512, 512, 16, 128, 1, 0, 3, 1, 1, False, False, 1.5),
    ("no_split_small_k", 2, 32, 64, 8, 200, 1, 4, 1, 1, 1, False, True, 2.0),
    ("groups2_mask_og4", 2, 64, 128, 4, 160, 2, 2, 2, 2, 4, True, False, 3.0),
    ("far_offsets_slow_taps", 1, 64, 64, 8, 256, 1, 3, 1, 1, 2, False, True, 90.0),
    ("cout_512_two_blocks", 1, 64, 512, 4, 300, 1, 1, 1, 1, 1, True, True, 2.0),
    # L_out = 256: tiles stay inside one batch row
    ("row_tiles_lout_256", 2, 32, 64, 9, 264, 1, 0, 1, 1, 1, False, False, 2.0),
    # L_out = 21: one 128-row tile spans 8 batch rows, the last tile is ragged
    ("short_rows_span_8_batches", 9, 64, 64, 8, 28, 1, 0, 1, 1, 1, True, False, 2.0),
    # two x windows per batch row do not fit beside N = 256 twice: row tiles instead
    ("flat_falls_back_to_rows", 2, 32, 256, 16, 300, 2, 0, 1, 1, 1, False, False, 2.0),
    # L_out = 1: one tile, its reduction split across a cluster of 8 CTAs
    ("lout_1_scalar_reduce", 2, 256, 64, 16, 16, 1, 0, 1, 1, 1, False, False, 2.0),
    # 24 and 21 tiles: clusters of 6 and 7 splits, so the 16 column chunks of a tile are
    # owned unevenly (3 or 2 per CTA)
    ("split6_uneven_chunk_owners", 37, 96, 256, 16, 128, 1, 0, 3, 1, 1, False, False, 1.5),
    ("split7_uneven_chunk_owners", 32, 112, 256, 16, 128, 1, 0, 3, 1, 1, True, False, 1.5),
]


@pytest.mark.parametrize("case", TF32_CASES, ids=[c[0] for c in TF32_CASES])
def test_tc_tf32_parity(case):
    name, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, sc = case
    L_out = oracle.out_length(L, K, s, p, d)
    w, t = W.small_case(31, B=B, C_in=Ci, C_out=Co, K=K, stride=s, padding=p, dilation=d,
                        groups=G, offset_groups=og, L_in=L, L_out=L_out, dtype="f32",
                        mask=mask, unconstrained=unc, off_scale=sc)
    td = to_dev(t)
    assert kernel_name(w, td) == "tcgen05_3xtf32", kernel_name(w, td)
    y = gpu_forward(w, td)
    assert dcn.dcn1d_device_status() == 0
    r = oracle_full(w, t)
    err = norm_err(y.double().cpu().numpy(), r)
    assert err <= TOL["f32"], (name, err)


def test_tf32_is_one_launch_without_workspace():
    """The fp32 tensor-core path (split-K included) needs no scratch: dcn1d_forward without
    any workspace runs it as one launch, bit for bit like a call given a workspace."""
    w = W.USAGE_F32.with_batch(2)
    td = to_dev(W.make_inputs(w, seed=2))
    assert dcn.dcn1d_forward_workspace_size(td["x"], td["offsets"], td["mask"], td["weight"],
                                            td["bias"], w.stride, w.padding, w.dilation,
                                            w.groups, w.offset_groups, w.unconstrained) == 0
    assert kernel_name(w, td) == "tcgen05_3xtf32"
    a = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"],
                          w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                          w.unconstrained, workspace=torch.empty(1 << 20, dtype=torch.uint8,
                                                                 device="cuda"))
    b = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"],
                          w.stride, w.padding, w.dilation, w.groups, w.offset_groups,
                          w.unconstrained, workspace=False)
    torch.cuda.synchronize()
    assert dcn.dcn1d_last_launch_count() == 1
    assert dcn.dcn1d_device_status() == 0
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_tf32_deterministic_across_calls():
    w = W.USAGE_F32.with_batch(3)
    td = to_dev(W.make_inputs(w, seed=5))
    a = gpu_forward(w, td)
    launches = dcn.dcn1d_last_launch_count()
    b = gpu_forward(w, td)
    torch.cuda.synchronize()
    assert launches == 1
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


# The three-product split reaches about fp32 accuracy; one TF32 product per term (or a
# tensor core that rounded, instead of truncating, the fp32 weight it reads as the high
# part) gives about 1e-4 on this shape.  The bound pins the split, not just the tolerance.
TF32_SPLIT_BOUND = 1e-5


@pytest.mark.parametrize("scale_low_bits", [False, True], ids=["plain", "low_bits_set"])
def test_tf32_three_products_reach_fp32_accuracy(scale_low_bits):
    w = W.USAGE_F32.with_batch(2)
    t = W.make_inputs(w, seed=11)
    if scale_low_bits:   # weights whose low mantissa bits are all populated
        t["weight"] = (t["weight"].double() * (1.0 + 2.0 ** -12)).float()
    td = to_dev(t)
    assert kernel_name(w, td) == "tcgen05_3xtf32"
    y = gpu_forward(w, td)
    assert dcn.dcn1d_device_status() == 0
    err = norm_err(y.double().cpu().numpy(), oracle_full(w, t))
    assert err <= TF32_SPLIT_BOUND, err


def test_tf32_split_sums_into_a_misaligned_output():
    """An output view that is only 4-byte aligned takes the one-at-a-time reduction; the
    result is the same bits as with an aligned output."""
    w = W.USAGE_F32.with_batch(2)
    td = to_dev(W.make_inputs(w, seed=13))
    ref = gpu_forward(w, td)
    buf = torch.full((ref.numel() + 1,), float("nan"), device="cuda")
    out = buf[1:].view(ref.shape)
    assert out.data_ptr() % 16 != 0
    y = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], td["weight"], td["bias"], w.stride,
                          w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained,
                          out=out)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    assert torch.equal(y.view(torch.int32), ref.view(torch.int32))
