"""The C-ABI library loads, exports every entry point include/moeq.h declares,
and its host-side validation rejects bad arguments before any device work.
CPU only: no call here reaches a kernel launch."""
import ctypes as C
import os
import re

import pytest

from quantised_expert_ffn_moe_b200 import build as moeq_build
from quantised_expert_ffn_moe_b200 import moeq, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    moeq_build.build()
    return moeq.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "moeq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    assert sorted(moeq.EXPORTS) == _declared()


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_version(L):
    assert moeq.version().startswith("moeq")


def _desc(**kw):
    d = dict(hidden=4096, inter=1024, n_experts=512, top_k=10, group_size=64, bits=4, has_shared=1)
    d.update(kw)
    return moeq.LayerDesc(*(d[n] for n in ("hidden", "inter", "n_experts", "top_k",
                                           "group_size", "bits", "has_shared")))


def test_workspace_size(L):
    d = _desc()
    one = moeq.workspace_size(d, 1)
    assert one > 0 and moeq.workspace_size(d, 4) - 256 == 4 * (one - 256)
    # h of the 11 active experts and the operand image of x (16 windows of
    # 256 eight-byte entries) are part of it
    assert one >= 11 * 1024 * 4 + 16 * 256 * 8
    assert moeq.workspace_size(d, 0) == 256


@pytest.mark.parametrize("bad", [dict(group_size=32), dict(bits=3), dict(hidden=100), dict(inter=0),
                                 dict(top_k=0), dict(top_k=33, n_experts=64), dict(top_k=9, n_experts=8),
                                 dict(n_experts=2048), dict(has_shared=2), dict(hidden=16384)])
def test_invalid_desc_rejected(L, bad):
    d = _desc(**bad)
    assert moeq.workspace_size(d, 1) == 0
    rc = L.moe_route(C.byref(d), C.c_void_p(16), 1, C.c_void_p(16), 0, None, C.c_void_p(16),
                     C.c_void_p(16), C.c_void_p(256), None)
    assert rc in (moeq.MOE_ERR_INVALID_ARG, moeq.MOE_ERR_UNSUPPORTED)
    assert moeq.last_error() != ""


def test_unsupported_vs_invalid(L):
    d = _desc(group_size=128)
    assert L.moe_route(C.byref(d), C.c_void_p(16), 1, C.c_void_p(16), 0, None, C.c_void_p(16),
                       C.c_void_p(16), C.c_void_p(256), None) == moeq.MOE_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected(L):
    d = _desc()
    ws = C.c_void_p(1 << 20)
    # NULL desc
    assert L.moe_route(None, C.c_void_p(16), 1, C.c_void_p(16), 0, None, C.c_void_p(16),
                       C.c_void_p(16), ws, None) == moeq.MOE_ERR_INVALID_ARG
    # misaligned x / router / workspace
    for x, wr, w in ((C.c_void_p(18), C.c_void_p(16), ws), (C.c_void_p(16), C.c_void_p(20), ws),
                     (C.c_void_p(16), C.c_void_p(16), C.c_void_p(300))):
        assert L.moe_route(C.byref(d), x, 1, wr, 0, None, C.c_void_p(16), C.c_void_p(16), w,
                           None) == moeq.MOE_ERR_INVALID_ARG
    # negative T
    assert L.moe_route(C.byref(d), C.c_void_p(16), -1, C.c_void_p(16), 0, None, C.c_void_p(16),
                       C.c_void_p(16), ws, None) == moeq.MOE_ERR_INVALID_ARG
    # bad router dtype
    assert L.moe_route(C.byref(d), C.c_void_p(16), 1, C.c_void_p(16), 7, None, C.c_void_p(16),
                       C.c_void_p(16), ws, None) == moeq.MOE_ERR_INVALID_ARG


def test_zero_tokens_is_a_no_op(L):
    d = _desc()
    assert L.moe_route(C.byref(d), None, 0, None, 0, None, None, None, C.c_void_p(256),
                       None) == moeq.MOE_OK


def test_expert_ffn_checks(L):
    d = _desc()
    st = moeq.SlotTable(C.c_void_p(4096).value, 512)
    sh = moeq.QExpert(*(moeq.QMat(16, 2, 2) for _ in range(3)))
    args = lambda dd, slots, shared: (C.byref(dd), C.c_void_p(16), 1, slots, shared, C.c_void_p(16),
                                      C.c_void_p(16), C.c_void_p(16), C.c_void_p(256), None)
    # entry point / bits mismatch
    assert L.moe_expert_ffn_q2(*args(d, C.byref(st), C.byref(sh))) == moeq.MOE_ERR_INVALID_ARG
    # shared required by has_shared
    assert L.moe_expert_ffn_q4(*args(d, C.byref(st), None)) == moeq.MOE_ERR_INVALID_ARG
    # shared given without has_shared
    assert L.moe_expert_ffn_q4(*args(_desc(has_shared=0), C.byref(st), C.byref(sh))) == moeq.MOE_ERR_INVALID_ARG
    # too few slots
    st2 = moeq.SlotTable(C.c_void_p(4096).value, 100)
    assert L.moe_expert_ffn_q4(*args(d, C.byref(st2), C.byref(sh))) == moeq.MOE_ERR_INVALID_ARG
    # misaligned shared codes
    sh2 = moeq.QExpert(moeq.QMat(24, 2, 2), moeq.QMat(16, 2, 2), moeq.QMat(16, 2, 2))
    assert L.moe_expert_ffn_q4(*args(d, C.byref(st), C.byref(sh2))) == moeq.MOE_ERR_INVALID_ARG


def test_layer_forward_rejects_out_overlapping_x(L):
    d = _desc()
    st = moeq.SlotTable(C.c_void_p(4096).value, 512)
    sh = moeq.QExpert(*(moeq.QMat(16, 2, 2) for _ in range(3)))
    x = 1 << 20
    rc = L.moe_layer_forward(C.byref(d), C.c_void_p(x), C.c_void_p(x), 1, C.c_void_p(16), 0, None,
                             C.byref(st), C.byref(sh), None, C.c_void_p(x + 64), None, None,
                             C.c_void_p(256), None)
    assert rc == moeq.MOE_ERR_INVALID_ARG and "overlap" in moeq.last_error()


def test_desc_matches_synth_shapes():
    d = moeq.make_desc(synth.DECODE_397B)
    assert (d.hidden, d.inter, d.n_experts, d.top_k, d.group_size, d.bits, d.has_shared) == \
        (4096, 1024, 512, 10, 64, 4, 1)


class _FakeSlots:
    """Host-side stand-in for moeq.DeviceSlots (pointers are never read for
    zero tokens or rejected calls)."""
    def __init__(self):
        self.struct = moeq.SlotTable(C.c_void_p(4096).value, 512)
        self.shared = moeq.QExpert(*(moeq.QMat(16, 2, 2) for _ in range(3)))


def test_python_wrappers_marshal_every_argument(L):
    """Each wrapper passes the argument list its entry point declares (a
    wrong count raises TypeError in ctypes): zero-token calls return before
    any device work."""
    import torch
    d = _desc()
    h = torch.zeros((0, 4096), dtype=torch.bfloat16)
    wr = torch.zeros((512, 4096), dtype=torch.bfloat16)
    ws = torch.zeros(4096, dtype=torch.uint8)
    ws = ws[(256 - ws.data_ptr() % 256) % 256:]
    slots = _FakeSlots()

    class _NullStream:  # the default stream, without touching CUDA
        cuda_stream = 0
    s = _NullStream()
    moeq.layer_forward(d, h, h, wr, slots, ws, out=torch.zeros_like(h), stream=s)
    moeq.layer_forward_normed(d, h, wr, slots, ws, 1e-6, out=torch.zeros_like(h), stream=s)
    moeq.rmsnorm(h, 1e-6, out=torch.zeros_like(h), stream=s)
    moeq.route(d, h, wr, ws, stream=s)
    with pytest.raises(moeq.MoeError):
        moeq.layer_forward_normed(d, h, wr, slots, ws, -1.0, out=torch.zeros_like(h), stream=s)


def test_layer_forward_normed_rejects_overlaps(L):
    d = _desc()
    st = moeq.SlotTable(C.c_void_p(4096).value, 512)
    sh = moeq.QExpert(*(moeq.QMat(16, 2, 2) for _ in range(3)))
    x = 1 << 20
    # out partially overlapping h
    rc = L.moe_layer_forward_normed(C.byref(d), C.c_void_p(x), 1, C.c_float(1e-6), C.c_void_p(16), 0, None,
                                    C.byref(st), C.byref(sh), None, C.c_void_p(x + 64), None, None, None,
                                    C.c_void_p(256), None)
    assert rc == moeq.MOE_ERR_INVALID_ARG and "overlap" in moeq.last_error()
    # x-hat copy overlapping h
    rc = L.moe_layer_forward_normed(C.byref(d), C.c_void_p(x), 1, C.c_float(1e-6), C.c_void_p(16), 0, None,
                                    C.byref(st), C.byref(sh), None, C.c_void_p(x), C.c_void_p(x + 4096), None,
                                    None, C.c_void_p(256), None)
    assert rc == moeq.MOE_ERR_INVALID_ARG and "overlap" in moeq.last_error()


def test_workspace_grows_by_the_prefill_area_from_64_tokens():
    """From 64 tokens on, 4-bit layers with hidden and inter multiples of 128
    take the expert-sorted GEMM path, whose area (sorted rows of x, h and y,
    tile list, per-expert counts) is added to the per-token blocks; 2-bit
    layers stay on the per-token path."""
    d4 = _desc()
    per_tok = moeq.workspace_size(d4, 2) - moeq.workspace_size(d4, 1)
    assert moeq.workspace_size(d4, 63) == 256 + 63 * per_tok
    extra = moeq.workspace_size(d4, 64) - (256 + 64 * per_tok)
    # at least the sorted fp16 x rows, fp16 h (two parts) and fp32 y rows of
    # the 64 x 11 (token, expert) pairs
    pairs = 64 * 11
    assert extra >= pairs * (4096 * 2 + 1024 * 2 * 2 + 4096 * 4)
    d2 = _desc(bits=2)
    per2 = moeq.workspace_size(d2, 2) - moeq.workspace_size(d2, 1)
    assert moeq.workspace_size(d2, 64) == 256 + 64 * per2
    odd = _desc(hidden=4096 + 64)  # hidden not a multiple of 128: per-token path
    per_odd = moeq.workspace_size(odd, 2) - moeq.workspace_size(odd, 1)
    assert moeq.workspace_size(odd, 100) == 256 + 100 * per_odd


def test_header_is_plain_c(tmp_path):
    """include/moeq.h compiles as C11 and as C++17 (plain C types only, no
    torch or CUDA types in the signatures)."""
    import subprocess
    src = tmp_path / "use.c"
    src.write_text('#include "moeq.h"\nint main(void) { moe_layer_desc d; (void)d; return (int)MOE_OK; }\n')
    inc = os.path.join(ROOT, "include")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, str(src)], check=True)
    cpp = tmp_path / "use.cpp"
    cpp.write_text(src.read_text())
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, str(cpp)], check=True)
