"""PackedDeformConv1d's forward as ONE kernel (GPU): the depthwise layer of the dc1d page's
PackedDeformConv1d example, whose predicted offsets and mask never leave the chip.

Each case asserts that the fused kernel runs, compares the layer's output with the oracle
layer (normwise, the dtype's tolerance) and with the two-launch path of the same call
(trunk kernel, predicted tensors through memory, depthwise forward).  Both paths form the
same fp32 sums in the same order and round the predicted tensors to the dtype at the same
point, so they must agree bit for bit.
"""
import numpy as np
import pytest
import torch

import deformable_convolution_dcn1d_b200 as dcn
import oracle
import workloads as W
from gpu_util import TOL, norm_err

pytestmark = pytest.mark.gpu

KEYS = ("x", "dw_weight", "dw_bias", "off_weight", "off_bias", "mask_weight", "mask_bias",
        "weight", "bias")

CASES = [
    # name, dtype, B, C, K, L_in, stride, padding, dilation, modulated, unconstrained, biases,
    # off_scale
    ("page_example_bf16", "bf16", 2, 64, 3, 304, 1, "same", 4, True, False, True, 2.0),
    ("c256_k3_d4_bf16", "bf16", 1, 256, 3, 1000, 1, "same", 4, True, False, True, 2.0),
    ("c128_k1_unmodulated_unc", "bf16", 2, 128, 1, 520, 1, (0, 0), 1, False, True, True,
     1.0),
    ("c64_k2_f16_nobias", "f16", 2, 64, 2, 264, 1, (1, 0), 3, True, False, False, 2.0),
    ("c64_k4_unmodulated_ragged", "bf16", 3, 64, 4, 200, 1, (2, 1), 2, False, False, True,
     2.0),
    # offsets of tens of positions: past the staged window's margin (global-memory taps)
    ("c192_k3_far_offsets_unc", "bf16", 2, 192, 3, 408, 1, (1, 1), 1, True, True, True, 60.0),
]
# A predicted offset whose bf16 rounding the GPU's fp32 trunk and the oracle's fp64 trunk
# take on different sides moves its tap by one bf16 step of the offset: 1/2 position at
# |offset| ~ 64, which on a random signal changes the sampled value by O(1).  Cases with
# offsets that large are checked against the two-launch path (bit for bit) and, for the
# sampling itself, by the exact probes of test_gpu_index_exact.py; the rest against the
# oracle within the dtype's tolerance.
ORACLE_CHECKED = {c[0] for c in CASES if c[-1] <= 3.0}


def _setup(case, seed=5):
    (name, dt, B, C, K, L, s, pad, d, mod, unc, biases, sc) = case
    pl, pr = dcn.resolve_padding(pad, K, s, d)
    L_out = oracle.out_length(L, K, s, (pl, pr), d)
    w, t = W.packed_case(seed, B=B, C_in=C, C_out=C, K=K, stride=s, padding=pl, dilation=d,
                         groups=C, offset_groups=C, L_in=L, L_out=L_out, dtype=dt,
                         modulated=mod, biases=biases, off_scale=sc)
    return w, t, pad, (pl, pr), unc


def _run(w, td, pad, unc, with_offsets):
    r = dcn.dcn1d_packed_forward(*[td[k] for k in KEYS], w.stride, pad, w.dilation, w.groups,
                                 w.offset_groups, unc, with_offsets=with_offsets)
    return r[0] if with_offsets else r


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fused_layer(case):
    w, t, pad, pads, unc = _setup(case)
    td = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
    args = ([td[k] for k in KEYS], w.stride, pad, w.dilation, w.groups, w.offset_groups, unc)
    assert dcn.dcn1d_packed_forward_kernel_name(*args[0], *args[1:]) == "packed_fused_tcgen05"
    two = dcn.dcn1d_packed_forward_kernel_name(*args[0], *args[1:], with_offsets=True)
    assert two.startswith("trunk_"), two
    y = _run(w, td, pad, unc, False)
    torch.cuda.synchronize()
    assert dcn.dcn1d_last_launch_count() == 1
    assert dcn.dcn1d_device_status() == 0
    y2 = _run(w, td, pad, unc, True)          # the two-launch path of the same layer
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    r, _, _ = oracle.packed_forward(*[t[k] for k in KEYS], w.stride, pads, w.dilation, w.groups,
                                    w.offset_groups, unc)
    err = norm_err(y.double().cpu().numpy(), r)
    print(f"{case[0]}: max_rel_err={err:.3e} vs the oracle layer")
    if case[0] in ORACLE_CHECKED:
        assert err <= TOL[w.dtype], (case[0], err)
    if two == "trunk_tcgen05+depthwise":   # the same sums in the same order
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), \
            (case[0], int((y != y2).sum()))


def test_fused_needs_no_workspace():
    w, t, pad, pads, unc = _setup(CASES[0])
    td = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
    from deformable_convolution_dcn1d_b200 import _binding as Bd
    out = torch.empty((w.B, w.C_out, w.L_out), dtype=td["x"].dtype, device="cuda")
    refs = [Bd._ref(Bd._desc(td[k])) for k in KEYS]
    lib = dcn.load()
    args = (w.stride, pads[0], pads[1], w.dilation, w.groups, w.offset_groups, int(unc))
    need = lib.dcn1d_packed_forward_workspace_size(*refs, *args, None, None,
                                                   Bd._ref(Bd._desc(out)))
    assert need == 0
    st = lib.dcn1d_packed_forward(*refs, *args, None, None, Bd._ref(Bd._desc(out)), None, 0,
                                  Bd._P(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    ref = _run(w, td, pad, unc, True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_packed_workload_full_size_sampled():
    """The bench's packed workload at full size, through the fused kernel: every channel of
    four 128-position windows against the oracle layer run on short slices of the signal,
    and the whole output bit for bit against the two-launch path."""
    w = W.PACKED_MODULATED_BF16
    t = W.make_packed_inputs(w, seed=0)
    td = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
    pad = (w.padding, w.padding)
    assert dcn.dcn1d_packed_forward_kernel_name(*[td[k] for k in KEYS], w.stride, pad,
                                                w.dilation, w.groups, w.offset_groups,
                                                w.unconstrained) == "packed_fused_tcgen05"
    y = _run(w, td, pad, w.unconstrained, False)
    y2 = _run(w, td, pad, w.unconstrained, True)
    torch.cuda.synchronize()
    assert dcn.dcn1d_device_status() == 0
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    # oracle on slices: outputs at l depend on x[l - 8 .. l + 8] only (K 3, dilation 4,
    # constrained taps), so a slice with 64 positions of margin reproduces them exactly
    rng = np.random.default_rng(3)
    yc = y.double().cpu().numpy()
    for b in (0, w.B - 1):
        for l0 in rng.integers(64, w.L_in - 256, 2):
            sl = dict(t)
            sl["x"] = t["x"][b:b + 1, :, l0 - 64:l0 + 192].contiguous()
            r, _, _ = oracle.packed_forward(*[sl[k] for k in KEYS], w.stride, pad, w.dilation,
                                            w.groups, w.offset_groups, w.unconstrained)
            got = yc[b, :, l0:l0 + 128]
            ref = r[0, :, 64:192]
            assert norm_err(got, ref) <= TOL["bf16"], (b, l0)
