"""Host-side tests of the PackedDeformConv1d entry points of the C ABI (no GPU): the size
and kernel-name queries, and every invalid argument rejected with its status code before
anything is launched."""
import ctypes

import pytest

import deformable_convolution_dcn1d_b200 as dcn
from test_abi_host import T

R = lambda t: None if t is None else ctypes.byref(t)  # noqa: E731


def valid(**over):
    """B2 C_in 4 C_out 6 K3 L16, s1 p(1,1) d1, groups 2, offset_groups 2 (J = 6), modulated."""
    B, Ci, Co, K, L, og = 2, 4, 6, 3, 16, 2
    J = og * K
    a = dict(x=T((B, Ci, L)), dw=T((Ci, 1, K)), dwb=T((Ci,)), ow=T((J, Ci, 1)), ob=T((J,)),
             mw=T((J, Ci)), mb=T((J,)), w=T((Co, Ci // 2, K)), b=T((Co,)), stride=1, pl=1,
             pr=1, dilation=1, groups=2, og=og, unc=0, off=T((B, og, L, K)),
             mask=T((B, og, L, K)), out=T((B, Co, L)))
    a.update(over)
    return a


def trunk(a):
    lib = dcn.load()
    return lib.dcn1d_packed_trunk(R(a["x"]), R(a["dw"]), R(a["dwb"]), R(a["ow"]), R(a["ob"]),
                                  R(a["mw"]), R(a["mb"]), a["stride"], a["pl"], a["pr"],
                                  a["dilation"], a["og"], R(a["off"]), R(a["mask"]), None)


def trunk_name(a):
    lib = dcn.load()
    r = lib.dcn1d_packed_trunk_kernel_name(R(a["x"]), R(a["dw"]), R(a["dwb"]), R(a["ow"]),
                                           R(a["ob"]), R(a["mw"]), R(a["mb"]), a["stride"],
                                           a["pl"], a["pr"], a["dilation"], a["og"], R(a["off"]),
                                           R(a["mask"]))
    return r.decode() if r else None


def layer_args(a):
    return (R(a["x"]), R(a["dw"]), R(a["dwb"]), R(a["ow"]), R(a["ob"]), R(a["mw"]), R(a["mb"]),
            R(a["w"]), R(a["b"]), a["stride"], a["pl"], a["pr"], a["dilation"], a["groups"],
            a["og"], a["unc"], R(a["off"]), R(a["mask"]), R(a["out"]))


def ws_size(a):
    return int(dcn.load().dcn1d_packed_forward_workspace_size(*layer_args(a)))


def layer(a, ws=None, ws_bytes=0):
    return dcn.load().dcn1d_packed_forward(*layer_args(a), ws, ws_bytes, None)


def test_queries_on_valid_arguments():
    a = valid()
    assert trunk_name(a) == "trunk_simt"   # fp32 takes the CUDA-core trunk
    assert trunk_name(valid(**{k: T(tuple(v.shape[:v.ndim]), dtype=1) for k, v in valid().items()
                               if isinstance(v, dcn.Dcn1dTensor)})) == "trunk_simt"  # C_in 4
    # outputs supplied: only the forward's own scratch (none for this shape)
    assert ws_size(a) == 0
    # predicted tensors in the workspace: one 256-byte aligned block per tensor
    n = 2 * 2 * 16 * 3 * 4
    assert ws_size(valid(off=None, mask=None)) == 2 * ((n + 255) // 256 * 256)
    assert ws_size(valid(off=None)) == (n + 255) // 256 * 256


def test_tensor_core_trunk_chosen_for_bf16_multiple_of_64_channels():
    B, Ci, K, L, og = 1, 128, 5, 64, 8
    J = og * K
    bf = dict(dtype=1)
    a = valid(x=T((B, Ci, L), **bf), dw=T((Ci, 1, K), **bf), dwb=T((Ci,), **bf),
              ow=T((J, Ci), **bf), ob=T((J,), **bf), mw=T((J, Ci), **bf), mb=T((J,), **bf),
              pl=2, pr=2, og=og, off=T((B, og, L, K), **bf), mask=T((B, og, L, K), **bf))
    assert trunk_name(a) == "trunk_tcgen05"
    assert trunk_name(dict(a, x=T((B, Ci - 64 + 8, L), **bf))) is None   # shapes disagree


BAD = [
    ("null x", dict(x=None), 1),
    ("null depthwise weight", dict(dw=None), 1),
    ("null offset head", dict(ow=None), 1),
    ("null offsets out", dict(off=None), 1),
    ("mask head without mask out", dict(mask=None), 1),
    ("mask out without mask head", dict(mw=None, mb=None), 4),
    ("mask bias without mask head", dict(mw=None, mask=None), 4),
    ("mixed dtype", dict(ow=T((6, 4, 1), dtype=1)), 2),
    ("unknown dtype", dict(mb=T((6,), dtype=9)), 2),
    ("depthwise weight not [C_in, 1, K]", dict(dw=T((4, 2, 3))), 3),
    ("offset head wrong width", dict(ow=T((5, 4, 1))), 3),
    ("offset head wrong trailing dim", dict(ow=T((6, 4, 2))), 3),
    ("mask head shape", dict(mw=T((6, 3))), 3),
    ("depthwise bias shape", dict(dwb=T((3,))), 3),
    ("offset bias shape", dict(ob=T((5,))), 3),
    ("offsets out L_out", dict(off=T((2, 2, 15, 3))), 3),
    ("mask out shape", dict(mask=T((2, 2, 16, 2))), 3),
    ("offset groups not dividing C_in", dict(og=3, ow=T((9, 4)), ob=T((9,)), mw=T((9, 4)),
                                             mb=T((9,)), off=T((2, 3, 16, 3)),
                                             mask=T((2, 3, 16, 3))), 4),
    ("stride 0", dict(stride=0), 4),
    ("negative right padding", dict(pr=-1), 4),
    ("L_out < 1", dict(x=T((2, 4, 1)), pl=0, pr=0, off=T((2, 2, 1, 3)),
                       mask=T((2, 2, 1, 3))), 4),
]


@pytest.mark.parametrize("name,over,code", BAD, ids=[b[0] for b in BAD])
def test_trunk_invalid_arguments(name, over, code):
    st = trunk(valid(**over))
    assert st == code, (name, dcn.dcn1d_status_string(st))
    assert dcn.dcn1d_last_launch_count() == 0


LAYER_BAD = [
    ("null weight", dict(w=None), 1),
    ("weight K differs from the trunk's", dict(w=T((6, 2, 5))), 3),
    ("out shape", dict(out=T((2, 6, 15))), 3),
    ("groups not dividing C_out", dict(groups=4, w=T((6, 1, 3))), 4),
    ("trunk arguments are checked too", dict(ow=T((5, 4))), 3),
]


@pytest.mark.parametrize("name,over,code", LAYER_BAD, ids=[b[0] for b in LAYER_BAD])
def test_layer_invalid_arguments(name, over, code):
    a = valid(**over)
    assert layer(a) == code, name
    assert ws_size(a) == -code
    assert dcn.dcn1d_last_launch_count() == 0


def test_layer_workspace_too_small_or_missing():
    a = valid(off=None, mask=None)
    assert layer(a) == 1                    # predicted tensors need a workspace
    assert layer(a, ctypes.c_void_p(0x10000), 256) == 4   # and one large enough
    assert dcn.dcn1d_last_launch_count() == 0
