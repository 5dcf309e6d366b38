"""Host-side checks of the C ABI: the library loads, exports every entry point the
header declares, and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

import ssd_sequence_mixing_b200 as ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20  # an aligned, never-dereferenced device address


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*[\w\s\*]*?\b(ssd_\w+)\s*\(", src, flags=re.M))
    return names


def test_library_exports_every_declared_entry_point():
    lib = ctypes.CDLL(ssd.LIB_PATH)
    decl = declared_functions()
    assert decl, "no declarations found"
    assert decl == set(ssd.EXPORTS), decl ^ set(ssd.EXPORTS)
    for name in decl:
        assert hasattr(lib, name), name


def shape(**kw):
    d = dict(batch=2, seqlen=300, nheads=4, headdim=64, dstate=128, ngroups=2, nseq=0, io_dtype=ssd.SSD_BF16)
    d.update(kw)
    return ssd.SsdShape(d["batch"], d["seqlen"], d["nheads"], d["headdim"], d["dstate"], d["ngroups"], d["nseq"],
                        d["io_dtype"], d.get("cu"))


def call(s, chunk=256, cu=None, **ptrs):
    p = {k: FAKE for k in ("x", "dt", "A", "B", "C", "y")}
    p.update(ptrs)
    v = lambda k: None if p.get(k) is None else ctypes.c_void_p(p[k])
    return ssd.library().ssd_forward(ctypes.byref(s), v("x"), v("dt"), v("A"), v("B"), v("C"), v("D"), v("init"),
                                     None if cu is None else ctypes.c_void_p(cu), chunk, v("y"), v("fin"), None)


@pytest.mark.parametrize("chunk", [0, 32, 100, 512])
def test_unsupported_chunk(chunk):
    assert call(shape(), chunk=chunk) == 2


def test_heads_not_multiple_of_groups():
    assert call(shape(nheads=6, ngroups=4)) == 2


@pytest.mark.parametrize("kw", [dict(headdim=257), dict(dstate=300), dict(nheads=70000, ngroups=1)])
def test_unsupported_sizes(kw):
    assert call(shape(**kw)) == 2


@pytest.mark.parametrize("kw", [dict(batch=-1), dict(nheads=0), dict(headdim=0), dict(dstate=0), dict(ngroups=0),
                                dict(io_dtype=7)])
def test_invalid_shape(kw):
    assert call(shape(**kw)) == 1


@pytest.mark.parametrize("missing", ["x", "dt", "A", "B", "C", "y"])
def test_null_required_pointer(missing):
    assert call(shape(), **{missing: None}) == 1


def test_null_shape():
    lib = ssd.library()
    assert lib.ssd_forward(None, *([None] * 8), 256, None, None, None) == 1


@pytest.mark.parametrize("which", ["x", "dt", "B", "y", "D", "init", "fin"])
def test_misaligned_pointer(which):
    assert call(shape(), **{which: FAKE + 4}) == 3


def test_packed_needs_single_row():
    assert call(shape(batch=2, nseq=3), cu=FAKE) == 1
    assert call(shape(batch=1, nseq=0), cu=FAKE) == 1


@pytest.mark.parametrize("vals", [[1, 5, 300], [0, 5, 299], [0, 7, 5, 300], [0, 400, 300]])
def test_bad_host_seqlens(vals):
    cu = torch.tensor(vals, dtype=torch.int32)
    s = shape(batch=1, nseq=len(vals) - 1, cu=cu.data_ptr())
    assert call(s, cu=FAKE) == 6


def test_status_strings_and_path_knob():
    lib = ssd.library()
    for code in range(7):
        assert lib.ssd_status_string(code)
    prev = ssd.set_path(ssd.PATH_SIMT)
    assert ssd.select_path(shape(), 256) == ssd.PATH_SIMT
    assert ssd.set_path(prev) == ssd.PATH_SIMT
    with pytest.raises(ssd.SsdError):
        ssd.set_path(9)
    assert ssd.select_path(shape(), 32) == -2


def test_workspace_bytes_grows_with_problem():
    old = ssd.set_path(ssd.PATH_SIMT)
    try:
        small = ssd.workspace_bytes(shape(seqlen=256), 256)
        big = ssd.workspace_bytes(shape(seqlen=4096), 256)
    finally:
        ssd.set_path(old)
    assert 0 < small < big
    # the SIMT path keeps one fp32 P x N state per chunk and head
    assert big >= 2 * 16 * 4 * 64 * 128 * 4


# ------------------------------------------------------------------ decode step
def call_decode(s, **ptrs):
    p = {k: FAKE for k in ("x", "dt", "A", "B", "C", "state", "y")}
    p.update(ptrs)
    v = lambda k: None if p.get(k) is None else ctypes.c_void_p(p[k])
    return ssd.library().ssd_decode_step(ctypes.byref(s), v("x"), v("dt"), v("A"), v("B"), v("C"), v("D"),
                                         v("state"), v("y"), None)


def test_decode_rejects_before_launch():
    assert call_decode(shape(seqlen=2)) == 1  # one token per row
    assert call_decode(shape(seqlen=1, nheads=0)) == 1
    assert call_decode(shape(seqlen=1, io_dtype=7)) == 1
    assert call_decode(shape(seqlen=1, dstate=6)) == 2  # N % 4
    assert call_decode(shape(seqlen=1, dstate=260)) == 2  # N > 256
    assert call_decode(shape(seqlen=1, nheads=6, ngroups=4)) == 2  # H % G
    for k in ("x", "dt", "A", "B", "C", "state", "y"):
        assert call_decode(shape(seqlen=1), **{k: None}) == 1, k
        assert call_decode(shape(seqlen=1), **{k: FAKE + 8}) == 3, k
    assert call_decode(shape(seqlen=1), D=FAKE + 4) == 3
    assert ssd.library().ssd_decode_step(None, *([None] * 8), None) == 1


def test_decode_empty_batch_is_a_no_op():
    assert call_decode(shape(seqlen=1, batch=0)) == 0


# ------------------------------------------------------------------ dt prologue
@pytest.mark.parametrize("bounds", [(-1.0, 1.0), (0.5, 0.1), (float("nan"), 1.0), (0.0, float("nan"))])
def test_dt_prologue_bad_bounds(bounds):
    pro = ssd.SsdDtPrologue(None, 1, bounds[0], bounds[1])
    p = {k: ctypes.c_void_p(FAKE) for k in ("x", "dt", "A", "B", "C", "y")}
    rc = ssd.library().ssd_forward_dt(ctypes.byref(shape()), ctypes.byref(pro), p["x"], p["dt"], p["A"], p["B"],
                                      p["C"], None, None, None, 256, p["y"], None, None)
    assert rc == 1


def test_dt_prologue_misaligned_bias():
    pro = ssd.SsdDtPrologue(FAKE + 4, 1, 0.0, float("inf"))
    p = {k: ctypes.c_void_p(FAKE) for k in ("x", "dt", "A", "B", "C", "y")}
    rc = ssd.library().ssd_forward_dt(ctypes.byref(shape()), ctypes.byref(pro), p["x"], p["dt"], p["A"], p["B"],
                                      p["C"], None, None, None, 256, p["y"], None, None)
    assert rc == 3


# ------------------------------------------------- block steps around the SSD
def test_conv_and_norm_reject_before_launch():
    lib = ssd.library()
    F = ctypes.c_void_p(FAKE)
    conv = lambda *a, **k: lib.ssd_causal_conv1d_silu(*a)
    assert conv(2, 10, 12, ssd.SSD_BF16, F, F, None, None, 0, F, None) == 2  # channels % 8
    assert conv(2, 10, 16, 9, F, F, None, None, 0, F, None) == 1
    assert conv(2, 10, 16, ssd.SSD_BF16, F, F, None, F, 3, F, None) == 1  # packed needs batch 1
    assert conv(1, 10, 16, ssd.SSD_BF16, None, F, None, None, 0, F, None) == 1
    assert conv(1, 10, 16, ssd.SSD_BF16, ctypes.c_void_p(FAKE + 4), F, None, None, 0, F, None) == 3
    assert conv(0, 10, 16, ssd.SSD_BF16, None, None, None, None, 0, None, None) == 0  # nothing to do
    norm = lib.ssd_gated_rmsnorm
    assert norm(4, 12, ssd.SSD_BF16, F, F, F, 1e-5, F, None) == 2  # dim % 8
    assert norm(4, 8200, ssd.SSD_BF16, F, F, F, 1e-5, F, None) == 2  # dim > 8192
    assert norm(4, 16, ssd.SSD_BF16, F, F, F, -1.0, F, None) == 1
    assert norm(4, 16, ssd.SSD_BF16, F, None, F, 1e-5, F, None) == 1
    assert norm(4, 16, ssd.SSD_BF16, F, F, ctypes.c_void_p(FAKE + 8), 1e-5, F, None) == 3
    assert norm(0, 16, ssd.SSD_BF16, None, None, None, 1e-5, None, None) == 0
