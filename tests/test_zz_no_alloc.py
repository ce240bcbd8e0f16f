"""pisa_precompute_noalloc against pisa_precompute, through the C ABI (needs a GPU).

Some callers of this library cannot allocate device memory: a plugin whose host framework owns every
device allocation and only hands it inputs and outputs, or a path that must not call cudaMalloc
because cudaMalloc can synchronise the device.  pisa_precompute_noalloc serves them by running the
pre-computation kernels with scratch taken from a fixed array in the library's own device memory.
This file checks it twice in a row, on different inputs, against the workspace entry point, for
every input type: both run the same deterministic kernels, so every statistic, operand copy and
scale must agree bit for bit.  It sits in a file of its own, named so that pytest collects it after
every other test.
"""
import ctypes

import pytest
import torch

from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

FIELDS = ("qbar", "kbar", "vsum", "hbar", "M", "kbar_op", "vsum_op", "hbar_op", "v_op", "vscale",
          "q8", "k8", "kbar8", "qscale", "kscale", "kbscale")


@pytest.mark.parametrize("dtype,head_dim", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16_fp8qk", 128)])
def test_noalloc_matches_workspace_entry_point_on_two_calls(dtype, head_dim):
    lib = C.lib()
    for seed in (11, 12):
        # 4 heads x 1200 tokens in blocks of 64 (a short last block): a few MB of scratch
        w = Workload("noalloc", 1, 4, (4, 15, 20), 0, head_dim, 64, 0.75, 0.5,
                     "fp32" if dtype == "fp32" else "bf16", seed=seed)
        q, k, v = (x.cuda() for x in make_qkv(w))
        shape = C.make_shape(1, 4, w.seq_len, head_dim, w.block, dtype)
        ref = C.alloc_stats(shape, "cuda")
        ws = C.alloc_workspace(shape, "cuda")
        C.pisa_precompute(shape, q, k, v, ref, ws)
        got = C.alloc_stats(shape, "cuda")
        got.buf.fill_(0x7F)
        stream = torch.cuda.current_stream().cuda_stream
        status = lib.pisa_precompute_noalloc(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             ctypes.byref(got.c), stream)
        assert status == C.PISA_OK, C.status_string(status)
        torch.cuda.synchronize()
        compared = 0
        for f in FIELDS:
            a, b = getattr(got, f), getattr(ref, f)
            assert (a is None) == (b is None), f
            if b is None:
                continue
            assert torch.equal(a, b), (dtype, seed, f)
            compared += 1
        assert compared >= (16 if dtype == "bf16_fp8qk" else 10 if dtype == "bf16" else 5)
        assert C.pisa_read_device_error(ws) == (C.PISA_OK, 0)


def _fake_stats():
    """Every pointer non-null and 16-byte aligned: passes argument checks, never dereferenced."""
    st = C.PisaStats()
    for name, _ in C.PisaStats._fields_:
        setattr(st, name, 256)
    return st


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = C.lib()
    shape = C.make_shape(1, 40, 75600, 128, 128, "bf16")      # needs ~97 MB of scratch
    st = _fake_stats()
    assert lib.pisa_precompute_noalloc(ctypes.byref(shape), 256, 256, 256, ctypes.byref(st), None) == \
        C.PISA_ERR_UNSUPPORTED


def test_noalloc_checks_arguments_first():
    lib = C.lib()
    small = C.make_shape(1, 2, 1024, 128, 64, "bf16")
    big = C.make_shape(1, 40, 75600, 128, 128, "bf16")
    st = _fake_stats()
    # a null or misaligned input is reported as such, whatever the shape's scratch needs
    for shape in (small, big):
        assert lib.pisa_precompute_noalloc(ctypes.byref(shape), None, 256, 256, ctypes.byref(st), None) == \
            C.PISA_ERR_INVALID_ARG
        assert lib.pisa_precompute_noalloc(ctypes.byref(shape), 256, 264, 256, ctypes.byref(st), None) == \
            C.PISA_ERR_INVALID_ARG
    bad = _fake_stats()
    bad.M = None
    assert lib.pisa_precompute_noalloc(ctypes.byref(small), 256, 256, 256, ctypes.byref(bad), None) == \
        C.PISA_ERR_INVALID_ARG
    odd = C.make_shape(1, 2, 1024, 96, 64, "bf16")
    assert lib.pisa_precompute_noalloc(ctypes.byref(odd), 256, 256, 256, ctypes.byref(st), None) == \
        C.PISA_ERR_UNSUPPORTED
