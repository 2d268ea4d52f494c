"""The algorithmic work the bench divides by (CPU only): flops and bytes per launch recounted
by brute force from the definitions on small shapes, and the roofline each kernel is held
to."""
import itertools

import pytest

import bench
import workloads as W


def small(**over):
    base = dict(B=2, C_in=6, C_out=4, K=3, stride=2, padding=1, dilation=2, groups=2,
                offset_groups=3, L_in=11, L_out=5, dtype="bf16", mask=True)
    base.update(over)
    w, _ = W.small_case(0, **base)
    return w


def brute_macs(w):
    """Multiply-adds of the forward's definition, one per (b, co, l, ci of co's group, k)."""
    cin_g = w.C_in // w.groups
    return sum(cin_g * w.K for _ in itertools.product(range(w.B), range(w.C_out),
                                                       range(w.L_out)))


@pytest.mark.parametrize("over", [{}, dict(groups=1, offset_groups=1, mask=False),
                                  dict(dtype="f32", C_in=4, C_out=4, groups=4,
                                       offset_groups=4)])
def test_forward_flops_and_bytes(over):
    w = small(**over)
    assert w.flops() == 2 * brute_macs(w)
    t = W.make_inputs(w, seed=0)
    es = 4 if w.dtype == "f32" else 2
    n = sum(v.numel() for v in t.values() if v is not None) + w.B * w.C_out * w.L_out
    assert w.algorithmic_bytes() == n * es


@pytest.mark.parametrize("modulated", [True, False])
def test_packed_flops_and_trunk_bytes(modulated):
    w, t = W.packed_case(0, B=2, C_in=8, C_out=8, K=3, stride=1, padding=2, dilation=2,
                         groups=8, offset_groups=4, L_in=20, L_out=20, dtype="bf16",
                         modulated=modulated)
    heads = 2 if modulated else 1
    J = w.offset_groups * w.K
    depthwise = w.B * w.L_out * w.C_in * w.K
    pointwise = w.B * w.L_out * heads * J * w.C_in
    deform = brute_macs(w)
    assert bench.packed_flops(w) == 2 * (depthwise + pointwise + deform)
    trunk_in = sum(t[k].numel() for k in ("x", "dw_weight", "dw_bias", "off_weight", "off_bias",
                                          "mask_weight", "mask_bias") if t[k] is not None)
    predicted = heads * w.B * w.offset_groups * w.L_out * w.K
    assert bench.packed_trunk_bytes(w) == (trunk_in + predicted) * 2
    # the fused layer: every input once, the output once, the predicted tensors not at all
    every_input = sum(v.numel() for v in t.values() if v is not None)
    assert bench.packed_layer_bytes(w) == (every_input + w.B * w.C_out * w.L_out) * 2


def test_each_kernel_is_held_to_its_own_roofline():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0,
             "source": "test"}
    w = small()
    assert bench.roofline_for("depthwise", w, peaks)[:3] == ("hbm", "GB/s", 6000.0)
    assert bench.roofline_for("tcgen05_bf16", w, peaks)[:3] == ("tensor", "TFLOP/s", 1600.0)
    assert bench.roofline_for("tcgen05_f16", w, peaks)[:3] == ("tensor", "TFLOP/s", 1600.0)
    bound, unit, peak = bench.roofline_for("tcgen05_3xtf32", w, peaks)[:3]
    assert (bound, unit) == ("tensor", "TFLOP/s")
    # the TF32 dense peak with the flops counted once, not divided by the three passes
    assert peak == pytest.approx(1600.0 * 1.1 / 2.25)
    assert bench.roofline_for("direct", w, peaks)[0] == "alu"


def test_default_line_is_the_largest_single_gpu_workload():
    """The bench's default line runs the workload with the most contraction work."""
    assert bench.DEFAULT_WORKLOAD == max(W.WORKLOADS.values(), key=lambda w: w.flops()).name
