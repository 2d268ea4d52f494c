"""Bit-exact sampling decisions inside every kernel the bench times (GPU).

The dc1d page's demo notebook treats an integer offset as an exact shift, and the floor
positions, clamps and neighbour choices of the sampling step must match the oracle bit for
bit.  The inputs of ``index_probe`` make each of those decisions show in the output: every
output is one sampled value, exact in the dtype, so the kernel's output must EQUAL the
oracle's result rounded to the dtype (``torch.equal``), with no tolerance.  Each case
asserts which kernel ran.  ``tests/test_index_probe_design.py`` shows, on the CPU, that the
same inputs catch a planted mistake in the floor, the clamp bounds or the neighbour choice.
"""
import zlib

import numpy as np
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
from index_probe import onehot_weight, probe_inputs, shifts_covering

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}

CASES = [
    # name, kernel, dtype, B, C_in, C_out, K, L_in, s, p, d, groups, og, mask, unc, near_int
    ("tc_k3_constrained", "tcgen05_bf16", "bf16", 2, 64, 192, 3, 264, 1, 0, 1, 1, 1,
     False, False, False),
    ("tc_k5_mask_og4_constrained", "tcgen05_bf16", "bf16", 2, 128, 256, 5, 200, 1, 2, 1, 1, 4,
     True, False, False),
    ("tc_k5_mask_og4_unconstrained", "tcgen05_bf16", "bf16", 2, 128, 256, 5, 200, 1, 2, 1, 1,
     4, True, True, False),
    ("tc_k9_strided_groups_unconstrained", "tcgen05_bf16", "bf16", 2, 128, 512, 9, 320, 2, 4,
     2, 2, 2, False, True, False),
    ("tc_k9_strided_groups_constrained", "tcgen05_bf16", "bf16", 1, 128, 512, 9, 320, 2, 4,
     2, 2, 2, True, False, False),
    ("tc_f16_k3_unconstrained", "tcgen05_f16", "f16", 2, 64, 192, 3, 264, 1, 1, 1, 1, 2,
     True, True, False),
    ("tc_k3_cout_512_two_blocks", "tcgen05_bf16", "bf16", 1, 64, 512, 3, 264, 1, 1, 1, 1, 1,
     False, True, False),
    ("tc_k16_d3_constrained", "tcgen05_bf16", "bf16", 2, 64, 128, 16, 128, 1, 0, 3, 1, 1,
     False, False, False),
    ("tc_k16_mask_og2_unconstrained", "tcgen05_bf16", "bf16", 2, 64, 64, 16, 200, 1, 8, 2, 1,
     2, True, True, False),
    ("tc_k5_mask_copy_mode_lin300", "tcgen05_bf16", "bf16", 2, 64, 128, 5, 300, 1, 2, 1, 1,
     2, True, True, False),
    ("tc_k9_strided_copy_mode_lin330", "tcgen05_bf16", "bf16", 1, 64, 128, 9, 330, 2, 4, 2, 1,
     1, False, False, False),
    ("tf32_k16_d3_constrained", "tcgen05_3xtf32", "f32", 2, 32, 512, 16, 128, 1, 0, 3, 1, 1,
     False, False, False),
    ("tf32_k4_strided_groups_mask_unconstrained", "tcgen05_3xtf32", "f32", 2, 64, 128, 4, 160,
     2, 2, 2, 2, 4, True, True, False),
    ("depthwise_bf16_k3_unconstrained", "depthwise", "bf16", 2, 64, 64, 3, 3001, 1, 64, 64,
     64, 64, False, True, False),
    ("depthwise_bf16_k5_mask_constrained", "depthwise", "bf16", 2, 32, 32, 5, 700, 2, 4, 2,
     32, 32, True, False, False),
    ("depthwise_f32_k3_mask_unconstrained", "depthwise", "f32", 2, 32, 32, 3, 900, 1, 8, 8,
     32, 32, True, True, True),
    ("direct_bf16_k6", "direct", "bf16", 2, 16, 32, 6, 90, 1, 2, 1, 1, 2, True, False,
     False),
]


def _forward(c, t, w, unc):
    """The forward through the C ABI on CUDA copies of t with weight w."""
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, _, _) = c
    td = {k: (v.to(DT[dt]).cuda() if v is not None else None) for k, v in t.items()}
    wd = w.to(DT[dt]).cuda()
    got = dcn.dcn1d_forward_kernel_name(td["x"], td["offsets"], td["mask"], wd, None, s, p, d,
                                        G, og, unc)
    assert got == kern, (name, got)
    y = dcn.dcn1d_forward(td["x"], td["offsets"], td["mask"], wd, None, s, p, d, G, og, unc)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    return y.cpu()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_every_sampled_value_bit_exact(case):
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, near_int) = case
    L_out = oracle.out_length(L, K, s, p, d)
    t = probe_inputs(B, Ci, L, L_out, K, d, og, mask, seed=zlib.crc32(name.encode()) % 1000,
                     near_integer=near_int)
    # the oracle reads exactly the values the kernel reads (the dtype's rounding of them)
    t = {k: (v.to(DT[dt]) if v is not None else None) for k, v in t.items()}
    shifts = ([0] if G == Ci == Co else shifts_covering(Co, Ci, K, G))
    for shift in shifts:
        if G == Ci == Co:      # depthwise: channel c reads tap (c + shift) mod K, every shift
            for sh in range(K):
                w = torch.zeros(Co, 1, K)
                w[torch.arange(Co), 0, (torch.arange(Co) + sh) % K] = 1.0
                _compare(case, t, w, unc)
        else:
            _compare(case, t, onehot_weight(Co, Ci, K, G, shift), unc)


def _compare(case, t, w, unc):
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, _, _) = case
    y = _forward(case, t, w, unc)
    r = oracle.forward(t["x"], t["offsets"], t["mask"], w.to(DT[dt]), None, s, p, d, G, og,
                       unc)
    ref = torch.from_numpy(np.ascontiguousarray(r)).to(DT[dt])
    if not torch.equal(y, ref):
        bad = (y.double() != ref.double()).nonzero()
        b, co, l = bad[0].tolist()
        raise AssertionError(f"{name}: {bad.shape[0]} outputs differ, first at "
                             f"(b={b}, co={co}, l={l}): {y[b, co, l].item()} vs "
                             f"{ref[b, co, l].item()}")


@pytest.mark.parametrize("case", [c for c in CASES if c[1] == "tcgen05_3xtf32"],
                         ids=lambda c: c[0])
def test_tf32_near_integer_offsets(case):
    """Offsets a few ulp from an integer: the sampled value then needs more bits than the
    three TF32 products carry (the low part of each operand is itself rounded to TF32,
    about 2^-22 relative), so the 3xTF32 kernel matches to that precision, not bit for
    bit.  An inconsistent floor or neighbour would be off by at least 1/4."""
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, _) = case
    L_out = oracle.out_length(L, K, s, p, d)
    t = probe_inputs(B, Ci, L, L_out, K, d, og, mask, seed=zlib.crc32(name.encode()) % 1000 + 1,
                     near_integer=True)
    for shift in shifts_covering(Co, Ci, K, G):
        w = onehot_weight(Co, Ci, K, G, shift)
        y = _forward(case, t, w, unc).double()
        r = torch.from_numpy(np.ascontiguousarray(oracle.forward(
            t["x"], t["offsets"], t["mask"], w, None, s, p, d, G, og, unc)))
        err = (y - r).abs().max().item()
        assert err <= 2.0 ** -18 * max(r.abs().max().item(), 1.0), (name, err)


def _packed_probe(C_in, C_out, K, L_in, stride, pads, dilation, groups, og, modulated, seed):
    """PackedDeformConv1d inputs whose predicted offsets are exact multiples of 1/4: the
    depthwise trunk passes x through from tap 0, the offset head reads a quarter of one
    trunk channel per output channel plus a bias from the probe's mixture, and the mask
    head (weights and bias zero) predicts exactly 1/2 everywhere."""
    from index_probe import probe_offsets, probe_x
    gen = torch.Generator().manual_seed(seed)
    J = og * K
    x = probe_x((2, C_in, L_in), gen)
    dw = torch.zeros(C_in, 1, K)
    dw[:, 0, 0] = 1.0
    off_w = torch.zeros(J, C_in)
    off_w[torch.arange(J), torch.randint(0, C_in, (J,), generator=gen)] = 0.25
    off_b = probe_offsets((1, og, 1, K), K, dilation, gen).reshape(J)
    t = {"x": x, "dw_weight": dw, "dw_bias": None, "off_weight": off_w, "off_bias": off_b,
         "mask_weight": torch.zeros(J, C_in) if modulated else None,
         "mask_bias": torch.zeros(J) if modulated else None}
    return t


PACKED = [
    # name, C_in, C_out, K, L_in, stride, padding, dilation, groups, og, modulated, forward
    ("packed_depthwise_page_example", 64, 64, 3, 300, 1, "same", 4, 64, 64, True, "depthwise"),
    # L_in a multiple of 8: without with_offsets this layer runs as one fused kernel
    ("packed_depthwise_fused_c128", 128, 128, 3, 304, 1, "same", 4, 128, 128, True,
     "depthwise"),
    ("packed_dense_og4_k5", 128, 128, 5, 264, 1, (2, 2), 1, 1, 4, True, "tcgen05_bf16"),
    ("packed_dense_unmodulated_k3", 64, 192, 3, 264, 1, (1, 1), 1, 1, 2, False,
     "tcgen05_bf16"),
]
# unconstrained forms of the depthwise layers (the probe's offsets include values past
# the window margin and far past the signal): name suffix "_unc"
PACKED += [(c[0] + "_unc",) + c[1:] for c in PACKED if c[0].startswith("packed_depthwise")]
KEYS = ("x", "dw_weight", "dw_bias", "off_weight", "off_bias", "mask_weight", "mask_bias",
        "weight", "bias")


@pytest.mark.parametrize("case", PACKED, ids=[c[0] for c in PACKED])
def test_packed_layer_bit_exact(case):
    name, Ci, Co, K, L, s, pad, d, G, og, modulated, fwd = case
    unc = name.endswith("_unc")
    pl, pr = dcn.resolve_padding(pad, K, s, d)
    t = _packed_probe(Ci, Co, K, L, s, (pl, pr), d, G, og, modulated,
                      seed=zlib.crc32(name.encode()) % 1000)
    t = {k: (v.to(torch.bfloat16) if v is not None else None) for k, v in t.items()}
    if G == Ci == Co:
        ws = []
        for sh in range(K):
            w = torch.zeros(Co, 1, K)
            w[torch.arange(Co), 0, (torch.arange(Co) + sh) % K] = 1.0
            ws.append(w)
    else:
        ws = [onehot_weight(Co, Ci, K, G, sh) for sh in shifts_covering(Co, Ci, K, G)]
    for w in ws:
        t["weight"] = w.to(torch.bfloat16)
        t["bias"] = None
        td = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
        y, pred = dcn.dcn1d_packed_forward(*[td[k] for k in KEYS], s, pad, d, G, og, unc,
                                           with_offsets=True)
        off, mask = pred if modulated else (pred, None)
        torch.cuda.synchronize()
        assert dcn.dcn1d_device_status() == 0
        kern = dcn.dcn1d_forward_kernel_name(td["x"], off, mask, td["weight"], None, s, pad, d,
                                             G, og, unc)
        assert kern == fwd, (name, kern)
        r, roff, _ = oracle.packed_forward(*[t[k] for k in KEYS], s, (pl, pr), d, G, og, unc)
        # the predicted offsets are exact too: compare them bit for bit first
        assert torch.equal(off.cpu(), torch.from_numpy(np.ascontiguousarray(roff)).to(
            torch.bfloat16)), name
        if modulated:
            assert bool((mask.cpu() == 0.5).all()), name
        ref = torch.from_numpy(np.ascontiguousarray(r)).to(torch.bfloat16)
        assert torch.equal(y.cpu(), ref), (name, int((y.cpu() != ref).sum()))
        # the same layer without the predicted tensors: one fused kernel where it applies
        y1 = dcn.dcn1d_packed_forward(*[td[k] for k in KEYS], s, pad, d, G, og, unc)
        torch.cuda.synchronize()
        assert dcn.dcn1d_device_status() == 0
        assert torch.equal(y1.cpu(), ref), (name, "fused", int((y1.cpu() != ref).sum()))


def test_nan_and_huge_offsets_stay_in_bounds():
    """An offset that is NaN, infinite or huge never reads outside the staged window: the
    call completes, no bounded wait gives up, outputs fed by a non-finite offset are NaN
    and every other output is exact (depthwise fp32 and bf16, the 16-bit tensor-core
    kernel, unconstrained)."""
    for kern, dt, B, C, Co, K, L, s, p, d, G, og in (
            ("depthwise", "f32", 1, 32, 32, 3, 600, 1, 8, 8, 32, 32),
            ("depthwise", "bf16", 1, 32, 32, 3, 600, 1, 8, 8, 32, 32),
            ("tcgen05_bf16", "bf16", 1, 64, 192, 3, 264, 1, 1, 1, 1, 1)):
        L_out = oracle.out_length(L, K, s, p, d)
        t = probe_inputs(B, C, L, L_out, K, d, og, False, seed=7)
        t = {k: (v.to(DT[dt]) if v is not None else None) for k, v in t.items()}
        off = t["offsets"].clone()
        flat = off.view(-1)
        bad = torch.tensor([5, 77, 130])            # elements (l*K + k) of group 0, batch 0
        flat[bad[0]] = float("nan")
        flat[bad[1]] = float("inf")
        flat[bad[2]] = -float("inf")
        flat[200] = 1.0e6                            # huge but finite: reads zeros
        if G == C == Co:
            w = torch.zeros(Co, 1, K)
            w[:, 0, 0] = 1.0
            w[:, 0, 1] = 1.0
            w[:, 0, 2] = 1.0
        else:
            w = onehot_weight(Co, C, K, G, 0)
        wd = w.to(DT[dt])
        td = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
        got = dcn.dcn1d_forward_kernel_name(td["x"], off.cuda(), None, wd.cuda(), None, s, p,
                                            d, G, og, True)
        assert got == kern, (kern, got)
        y = dcn.dcn1d_forward(td["x"], off.cuda(), None, wd.cuda(), None, s, p, d, G, og,
                              True)
        torch.cuda.synchronize()
        assert dcn.dcn1d_device_status() == 0
        y = y.cpu().double()
        # which outputs read a non-finite offset (b = 0, offset group 0, l = e // K): in
        # the depthwise kernel channel 0 only (one channel per offset group); in the
        # contraction every output channel at l, since a zero weight times NaN is NaN
        hit = torch.zeros_like(y, dtype=torch.bool)
        for e in bad.tolist():
            if G == C == Co:
                hit[0, 0, e // K] = True
            else:
                hit[0, :, e // K] = True
        assert torch.isnan(y[hit]).all(), kern
        # every other output matches the oracle run with those offsets replaced by 0 (they
        # feed no other output); the huge one is kept (the oracle handles it)
        off0 = off.clone()
        off0.view(-1)[bad] = 0.0
        r = torch.from_numpy(np.ascontiguousarray(oracle.forward(
            t["x"], off0, None, wd, None, s, p, d, G, og, True))).double()
        r = r.to(DT[dt]).double()
        assert torch.equal(y[~hit], r[~hit]), kern
