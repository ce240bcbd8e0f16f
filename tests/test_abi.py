"""Host-side checks of the C ABI: the library loads, exports every declared symbol, and rejects
invalid arguments before touching the GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

from piecewise_approximate_attention_b200 import _lib as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    import glob
    src = "".join(open(f).read() for f in glob.glob(os.path.join(ROOT, "include", "*.h")))
    return sorted(set(re.findall(r"PISA_API\s+[\w\s\*]*?\b(pisa_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = C.lib()
    names = _declared()
    assert len(names) >= 12
    assert set(names) == set(C.SYMBOLS)
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_blocks():
    assert C.lib().pisa_abi_version() == 7
    assert C.pisa_num_blocks(32760, 64) == 512
    assert C.pisa_num_blocks(75600, 128) == 591
    assert C.pisa_num_blocks(1, 64) == 1
    assert C.pisa_num_blocks(0, 64) == -1
    assert C.pisa_num_blocks(10, 0) == -1


def test_status_strings():
    for s in range(5):
        assert C.status_string(s)
    assert "unknown" in C.status_string(99)


def _shape(**kw):
    base = dict(batch=1, heads=2, seq_len=1000, head_dim=128, block=64, dtype="bf16", softmax_scale=1.0)
    base.update(kw)
    return C.make_shape(**base)


def test_stats_bytes_and_carve_are_host_only():
    sh = _shape()
    n0 = C.pisa_stats_bytes(sh, False)
    n1 = C.pisa_stats_bytes(sh, True)
    nb = 16
    assert n1 - n0 >= nb * 128 * 128 * (4 + 2)       # H (fp32) and its bf16 difference copy
    st = C.PisaStats()
    base = 1 << 20      # never dereferenced: carving is pointer arithmetic
    assert C.lib().pisa_stats_carve(ctypes.byref(sh), base, n1, 1, ctypes.byref(st)) == C.PISA_OK
    ptrs = [st.qbar, st.kbar, st.vsum, st.hbar, st.M, st.H, st.kbar_op, st.vsum_op, st.hbar_op, st.v_op, st.vscale,
            st.hdiff_op]
    assert all(p and p % 256 == 0 and base <= p < base + n1 for p in ptrs)
    assert len(set(ptrs)) == len(ptrs)
    assert C.lib().pisa_stats_carve(ctypes.byref(sh), base + 16, n1, 1, ctypes.byref(st)) == C.PISA_ERR_INVALID_ARG
    assert C.lib().pisa_stats_carve(ctypes.byref(sh), base, n1 - 1, 1, ctypes.byref(st)) == C.PISA_ERR_INVALID_ARG
    assert C.pisa_workspace_bytes(sh) >= 256 + 2 * 1 * 128 * 128 * 4
    # per-block mode: status word, per-row offsets and 1/D_t, the fp32 output
    assert C.pisa_perblock_workspace_bytes(sh) >= 256 + 2 * 1000 * 8 + 2 * 1000 * 128 * 4
    assert C.pisa_perblock_workspace_bytes(sh) >= C.pisa_workspace_bytes(sh)
    # fp32 mode needs no tensor-core operand copies
    f32 = _shape(dtype="fp32")
    st32 = C.PisaStats()
    n32 = C.pisa_stats_bytes(f32, False)
    assert C.lib().pisa_stats_carve(ctypes.byref(f32), base, n32, 0, ctypes.byref(st32)) == C.PISA_OK
    assert not st32.kbar_op and not st32.v_op and not st32.vscale and n32 < n0
    # without H there is no per-block operand copy; fp32 keeps H but has no operand copies
    st0 = C.PisaStats()
    assert C.lib().pisa_stats_carve(ctypes.byref(sh), base, n0, 0, ctypes.byref(st0)) == C.PISA_OK
    assert not st0.H and not st0.hdiff_op
    n32h = C.pisa_stats_bytes(f32, True)
    assert C.lib().pisa_stats_carve(ctypes.byref(f32), base, n32h, 1, ctypes.byref(st32)) == C.PISA_OK
    assert st32.H and not st32.hdiff_op
    assert not st0.q8 and not st0.qscale
    # e4m3 logits: operand copies plus the e4m3 copies and their scales
    f8 = _shape(dtype="bf16_fp8qk")
    n8 = C.pisa_stats_bytes(f8, False)
    st8 = C.PisaStats()
    assert C.lib().pisa_stats_carve(ctypes.byref(f8), base, n8, 0, ctypes.byref(st8)) == C.PISA_OK
    f8ptrs = [st8.q8, st8.k8, st8.kbar8, st8.qscale, st8.kscale, st8.kbscale, st8.kbar_op, st8.v_op]
    assert all(p and p % 256 == 0 for p in f8ptrs) and len(set(f8ptrs)) == len(f8ptrs)
    assert n8 - n0 >= 2 * 2 * 1000 * 128 + 2 * 16 * 128 + 2 * 1000 * 4


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=96), C.PISA_ERR_UNSUPPORTED),
    (dict(block=32), C.PISA_ERR_UNSUPPORTED),
    (dict(seq_len=0), C.PISA_ERR_INVALID_ARG),
    (dict(batch=0), C.PISA_ERR_INVALID_ARG),
    (dict(dtype=7), C.PISA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), C.PISA_ERR_INVALID_ARG),
    (dict(softmax_scale=0.0), C.PISA_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), C.PISA_ERR_INVALID_ARG),
    (dict(seq_len=64 * 4097), C.PISA_ERR_UNSUPPORTED),
    (dict(dtype=3), C.PISA_ERR_INVALID_ARG),
    (dict(dtype="bf16_fp8qk", head_dim=64), C.PISA_ERR_UNSUPPORTED),
])
def test_bad_shapes_rejected(kw, expect):
    sh = _shape(**kw)
    st = C.PisaStats()
    assert C.lib().pisa_precompute(ctypes.byref(sh), 16, 16, 16, ctypes.byref(st), 16, 1 << 30, None) == expect
    assert C.lib().pisa_precompute_zeroth_order(ctypes.byref(sh), 16, 16, 16, ctypes.byref(st), 16, 1 << 30,
                                                None) == expect
    assert C.pisa_stats_bytes(sh, False) == 0
    assert C.pisa_workspace_bytes(sh) == 0
    assert C.pisa_perblock_workspace_bytes(sh) == 0


def _fake_stats(sh):
    st = C.PisaStats()
    n = C.pisa_stats_bytes(sh, False)
    assert C.lib().pisa_stats_carve(ctypes.byref(sh), 1 << 24, n, 0, ctypes.byref(st)) == C.PISA_OK
    return st


def test_invalid_arguments_rejected_without_launch():
    L = C.lib()
    sh = _shape()
    st = _fake_stats(sh)
    ws = C.pisa_workspace_bytes(sh)
    P = 1 << 28
    bs = ctypes.byref(sh)
    # null / misaligned tensors
    assert L.pisa_precompute(bs, None, P, P, ctypes.byref(st), P, ws, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_precompute(bs, P + 4, P, P, ctypes.byref(st), P, ws, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_precompute(bs, P, P, P, ctypes.byref(st), P, ws - 1, None) == C.PISA_ERR_INVALID_ARG
    bad = C.PisaStats.from_buffer_copy(st)
    bad.kbar_op = None
    assert L.pisa_precompute(bs, P, P, P, ctypes.byref(bad), P, ws, None) == C.PISA_ERR_INVALID_ARG
    # the zeroth-order pre-computation checks the same arguments
    Z = L.pisa_precompute_zeroth_order
    assert Z(bs, None, P, P, ctypes.byref(st), P, ws, None) == C.PISA_ERR_INVALID_ARG
    assert Z(bs, P + 4, P, P, ctypes.byref(st), P, ws, None) == C.PISA_ERR_INVALID_ARG
    assert Z(bs, P, P, P, ctypes.byref(st), P, ws - 1, None) == C.PISA_ERR_INVALID_ARG
    assert Z(bs, P, P, P, ctypes.byref(st), None, ws, None) == C.PISA_ERR_INVALID_ARG
    assert Z(bs, P, P, P, ctypes.byref(bad), P, ws, None) == C.PISA_ERR_INVALID_ARG
    # routing arguments
    assert L.pisa_route(bs, ctypes.byref(st), 17, 0.5, P, None, None, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_route(bs, ctypes.byref(st), -1, 0.5, P, None, None, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_route(bs, ctypes.byref(st), 4, -0.1, P, None, None, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_route(bs, ctypes.byref(st), 4, float("inf"), P, None, None, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_route(bs, ctypes.byref(st), 4, 0.5, None, None, None, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_route(bs, ctypes.byref(st), 4, 0.5, P + 8, None, None, None) == C.PISA_ERR_INVALID_ARG
    # attention arguments
    att = lambda keep, mode, sel=P, o=P, wsb=ws: L.pisa_attention(bs, P, P, P, ctypes.byref(st), sel, None, keep,
                                                                  mode, o, P, wsb, None)
    assert att(4, 3) == C.PISA_ERR_INVALID_ARG
    assert att(4, -1) == C.PISA_ERR_INVALID_ARG
    # the per-block first-order mode needs the per-block operand copy in the stats and the larger
    # workspace
    assert att(4, C.PISA_MODE_PER_BLOCK) == C.PISA_ERR_INVALID_ARG
    sth = C.PisaStats()
    nh = C.pisa_stats_bytes(sh, True)
    assert L.pisa_stats_carve(bs, 1 << 24, nh, 1, ctypes.byref(sth)) == C.PISA_OK
    assert sth.hdiff_op
    assert L.pisa_attention(bs, P, P, P, ctypes.byref(sth), P, None, 4, C.PISA_MODE_PER_BLOCK, P, P, ws,
                            None) == C.PISA_ERR_INVALID_ARG
    assert att(0, C.PISA_MODE_EXACT_ONLY) == C.PISA_ERR_INVALID_ARG
    assert att(17, C.PISA_MODE_PISA) == C.PISA_ERR_INVALID_ARG
    assert att(4, C.PISA_MODE_PISA, sel=None) == C.PISA_ERR_INVALID_ARG
    assert att(4, C.PISA_MODE_PISA, o=None) == C.PISA_ERR_INVALID_ARG
    assert att(4, C.PISA_MODE_PISA, wsb=100) == C.PISA_ERR_INVALID_ARG
    code = ctypes.c_int32()
    assert L.pisa_read_device_error(None, ctypes.byref(code), None) == C.PISA_ERR_INVALID_ARG
    # e4m3 logits need their copies in the stats, and do not combine with the per-block mode
    f8 = _shape(dtype="bf16_fp8qk")
    st8 = _fake_stats(f8)
    b8 = ctypes.byref(f8)
    ws8 = C.pisa_perblock_workspace_bytes(f8)
    assert L.pisa_attention(b8, P, P, P, ctypes.byref(st8), P, None, 4, C.PISA_MODE_PER_BLOCK, P, P, ws8,
                            None) == C.PISA_ERR_UNSUPPORTED
    bad8 = C.PisaStats.from_buffer_copy(st8)
    bad8.kscale = None
    assert L.pisa_attention(b8, P, P, P, ctypes.byref(bad8), P, None, 4, C.PISA_MODE_PISA, P, P, ws8,
                            None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_precompute(b8, P, P, P, ctypes.byref(bad8), P, ws8, None) == C.PISA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(C, "_lib", None)
    monkeypatch.setattr(C, "_LIB_PATH", "/nonexistent/libpisa_b200.so")
    with pytest.raises(RuntimeError, match="not built"):
        C.lib()


def test_testing_hook_rejects_unknown_fault():
    assert C.lib().pisa_testing_set_attention_fault(7, 0) == C.PISA_ERR_INVALID_ARG
    assert C.lib().pisa_testing_set_attention_fault(0, 0) == C.PISA_OK
    # the pre-computation hook takes its own fault code only
    assert C.lib().pisa_testing_set_precompute_fault(1, 0) == C.PISA_ERR_INVALID_ARG
    assert C.lib().pisa_testing_set_precompute_fault(7, 0) == C.PISA_ERR_INVALID_ARG
    assert C.lib().pisa_testing_set_precompute_fault(0, 0) == C.PISA_OK


def test_reordering_entry_points_validate_without_launch():
    L = C.lib()
    P = 1 << 28
    # gather/scatter: null, misaligned, bad sizes, overlapping buffers
    assert L.pisa_permute_rows(None, P, P, 2, 100, 256, 0, 0, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_permute_rows(P + 8, P * 2, P * 3, 2, 100, 256, 0, 0, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_permute_rows(P, P * 2, P * 3, 2, 100, 200, 0, 0, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_permute_rows(P, P * 2, P * 3, 0, 100, 256, 0, 0, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_permute_rows(P, P * 2, P * 3, 2, 0, 256, 0, 0, None) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_permute_rows(P, P + 256, P * 3, 2, 100, 256, 0, 1, None) == C.PISA_ERR_INVALID_ARG
    # axis permutation: a permutation of "thw" is required
    out = (ctypes.c_int32 * 64)()
    for bad in (b"thh", b"th", b"thwx", b"abc", b""):
        assert L.pisa_axis_permutation(2, 2, 3, 0, bad, out, 64) == C.PISA_ERR_INVALID_ARG, bad
    assert L.pisa_axis_permutation(2, 2, 3, -1, b"thw", out, 64) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_axis_permutation(0, 2, 3, 0, b"thw", out, 64) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_axis_permutation(2, 2, 3, 0, b"thw", None, 64) == C.PISA_ERR_INVALID_ARG
    assert L.pisa_axis_permutation(2, 2, 3, 4, b"wth", out, 15) == C.PISA_ERR_INVALID_ARG   # needs 16
    assert L.pisa_axis_permutation(2, 2, 3, 4, b"wth", out, 16) == C.PISA_OK
    got = list(out[:16])
    assert sorted(got) == list(range(16)) and got[12:] == [12, 13, 14, 15]


def test_headers_are_plain_c_and_the_library_links_from_c(tmp_path):
    """tests/c/abi_consumer.c: the public headers compile as strict C99 and a C program linked
    against the library gets the same host-only answers as the binding (no GPU, no Python)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    libdir = os.path.dirname(C._LIB_PATH)
    exe = str(tmp_path / "abi_consumer")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", libdir, "-lpisa_b200",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr
    assert "c consumer ok: abi 7" in res.stdout


def test_precompute_route_checks_its_flags():
    L = C.lib()
    sh = _shape()
    st = _fake_stats(sh)
    ws = C.pisa_workspace_bytes(sh)
    P = 1 << 28
    for flags in (2, -1, 3):
        assert L.pisa_precompute_route(ctypes.byref(sh), P, P, P, ctypes.byref(st), 4, 0.5, P, None, None, P, ws, flags,
                                       None) == C.PISA_ERR_INVALID_ARG
    # the route arguments are checked as by pisa_route, before anything is enqueued
    assert L.pisa_precompute_route(ctypes.byref(sh), P, P, P, ctypes.byref(st), 17, 0.5, P, None, None, P, ws, 0,
                                   None) == C.PISA_ERR_INVALID_ARG
