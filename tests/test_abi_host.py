"""Host-side tests of the C ABI (no GPU): the library loads, exports every symbol the
header declares, computes L_out like the oracle, and rejects every invalid argument with
its status code before launching anything."""
import ctypes
import os
import re

import pytest

import deformable_convolution_dcn1d_b200 as dcn
import oracle
from conftest import ROOT

FAKE = 0x10000   # a non-NULL placeholder pointer: validation never dereferences it


def header_functions():
    src = open(os.path.join(ROOT, "include", "dcn1d.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dcn1d_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = dcn.load()
    names = header_functions()
    assert len(names) >= 6
    for n in names:
        assert hasattr(lib, n), n
    assert {s[0] for s in dcn.SIGNATURES} == set(names)


def test_out_length_matches_oracle():
    for L_in in (1, 3, 16, 100, 16000):
        for K in (1, 2, 3, 9, 16):
            for s in (1, 2, 3):
                for p in (0, 1, 4, 64):
                    for d in (1, 2, 3, 64):
                        assert dcn.dcn1d_out_length(L_in, K, s, p, d) == \
                            oracle.out_length(L_in, K, s, p, d)
    assert dcn.dcn1d_out_length(0, 3, 1, 0, 1) == -1
    assert dcn.dcn1d_out_length(8, 3, 0, 0, 1) == -1
    assert dcn.dcn1d_out_length(8, 3, 1, -1, 1) == -1
    assert dcn.dcn1d_out_length(2, 5, 1, 0, 1) == -1
    assert dcn.dcn1d_out_length(1 << 40, 3, 1, 0, 1) == -1


def test_status_strings():
    for code, name in dcn._binding.STATUS.items():
        assert dcn.dcn1d_status_string(code) == name
    assert dcn.dcn1d_status_string(12345) == "DCN1D_UNKNOWN_STATUS"


def T(shape, dtype=0, data=FAKE):
    d = dcn.Dcn1dTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    for i, s in enumerate(shape):
        d.shape[i] = s
    return d


def valid(**over):
    """A valid argument set (B2 Ci4 Co6 K3 L16, s1 p1 d1, groups 2, og 2) as a dict."""
    B, Ci, Co, K, L, s, p, d, G, og = 2, 4, 6, 3, 16, 1, 1, 1, 2, 2
    L_out = 16
    a = dict(x=T((B, Ci, L)), off=T((B, og, L_out, K)), mask=None, w=T((Co, Ci // G, K)),
             bias=T((Co,)), stride=s, padding=p, dilation=d, groups=G, og=og, unc=0,
             out=T((B, Co, L_out)))
    a.update(over)
    return a


def call(a):
    lib = dcn.load()
    r = lambda t: None if t is None else ctypes.byref(t)
    st = lib.dcn1d_forward(r(a["x"]), r(a["off"]), r(a["mask"]), r(a["w"]), r(a["bias"]),
                           a["stride"], a["padding"], a["dilation"], a["groups"], a["og"],
                           a["unc"], r(a["out"]), None)
    name = lib.dcn1d_forward_kernel_name(r(a["x"]), r(a["off"]), r(a["mask"]), r(a["w"]),
                                         r(a["bias"]), a["stride"], a["padding"], a["dilation"],
                                         a["groups"], a["og"], a["unc"], r(a["out"]))
    return st, name


def test_valid_arguments_pick_a_kernel():
    lib = dcn.load()
    r = lambda t: None if t is None else ctypes.byref(t)
    a = valid()
    name = lib.dcn1d_forward_kernel_name(r(a["x"]), r(a["off"]), r(a["mask"]), r(a["w"]),
                                         r(a["bias"]), a["stride"], a["padding"], a["dilation"],
                                         a["groups"], a["og"], a["unc"], r(a["out"]))
    assert name is not None and len(name) > 0


BAD = [
    ("null x", dict(x=None), 1),
    ("null x data", dict(x=T((2, 4, 16), data=None)), 1),
    ("null offsets", dict(off=None), 1),
    ("null weight", dict(w=None), 1),
    ("null out", dict(out=None), 1),
    ("unknown dtype", dict(x=T((2, 4, 16), dtype=7)), 2),
    ("mixed dtype", dict(w=T((6, 2, 3), dtype=1)), 2),
    ("mixed mask dtype", dict(mask=T((2, 2, 16, 3), dtype=1)), 2),
    ("x ndim", dict(x=T((2, 4, 16, 1))), 3),
    ("offsets ndim", dict(off=T((2, 2, 48))), 3),
    ("weight channels", dict(w=T((6, 3, 3))), 3),
    ("offsets L_out mismatch", dict(off=T((2, 2, 15, 3))), 3),
    ("offsets K mismatch", dict(off=T((2, 2, 16, 2))), 3),
    ("offsets groups mismatch", dict(off=T((2, 1, 16, 3))), 3),
    ("offsets batch mismatch", dict(off=T((1, 2, 16, 3))), 3),
    ("mask shape", dict(mask=T((2, 2, 16, 2))), 3),
    ("bias shape", dict(bias=T((5,))), 3),
    ("out shape", dict(out=T((2, 6, 15))), 3),
    ("negative extent", dict(x=T((2, 4, -16))), 3),
    ("stride 0", dict(stride=0), 4),
    ("negative padding", dict(padding=-1), 4),
    ("dilation 0", dict(dilation=0), 4),
    ("groups 0", dict(groups=0), 4),
    ("groups not dividing C_out", dict(groups=4, w=T((6, 1, 3))), 4),
    ("offset_groups not dividing C_in", dict(og=3, off=T((2, 3, 16, 3))), 4),
    ("L_out < 1", dict(x=T((2, 4, 1)), w=T((6, 2, 5)), padding=0, off=T((2, 2, 1, 5)),
                       out=T((2, 6, 1))), 4),
    ("length past 2^24", dict(x=T((1, 4, 1 << 24)), off=T((1, 2, 1 << 24, 3)),
                              out=T((1, 6, 1 << 24))), 5),
    ("tensor past 2^31 elements", dict(x=T((1 << 8, 4096, 1 << 12)), off=T((1 << 8, 2, 1 << 12, 3)),
                                       out=T((1 << 8, 6, 1 << 12)), w=T((6, 2048, 3)), groups=2), 5),
]


@pytest.mark.parametrize("name,over,code", BAD, ids=[b[0] for b in BAD])
def test_invalid_arguments_return_status_and_launch_nothing(name, over, code):
    st, kname = call(valid(**over))
    assert st == code, (name, dcn.dcn1d_status_string(st))
    assert kname is None
    assert dcn.dcn1d_last_launch_count() == 0


def test_empty_batch_is_ok_and_launches_nothing():
    st, kname = call(valid(x=T((0, 4, 16), data=None), off=T((0, 2, 16, 3), data=None),
                           out=T((0, 6, 16), data=None)))
    assert st == 0
    assert dcn.dcn1d_last_launch_count() == 0


def test_sample_index_invalid_arguments():
    lib = dcn.load()
    off = T((2, 2, 16, 3))
    f = lambda o, L, s, p, d, i0=FAKE, fr=FAKE: lib.dcn1d_sample_index(
        None if o is None else ctypes.byref(o), L, s, p, d, 0, i0, fr, None)
    assert f(None, 16, 1, 1, 1) == 1
    assert f(off, 16, 1, 1, 1, i0=None) == 1
    assert f(T((2, 2, 16, 3), dtype=5), 16, 1, 1, 1) == 2
    assert f(T((2, 2, 48)), 16, 1, 1, 1) == 3
    assert f(off, 16, 0, 1, 1) == 4
    assert f(off, 16, 1, 1, 1 << 25) == 5
    assert f(off, 17, 1, 1, 1) == 3          # L_out 17 != 16
    assert f(T((0, 2, 16, 3), data=None), 16, 1, 1, 1) == 0
