"""pisa_precompute_noalloc against pisa_precompute, through the C ABI (needs a GPU).

Some callers of this library cannot allocate device memory: a plugin whose host framework owns every
device allocation and only hands it inputs and outputs, or a path that must not call cudaMalloc
because cudaMalloc can synchronise the device.  pisa_precompute_noalloc serves them by running the
pre-computation kernels with scratch taken from a fixed array in the library's own device memory.
This file checks it twice in a row, on different inputs, against the workspace entry point.  It sits
in a file of its own, named so that pytest collects it after every other test.
"""
import ctypes

import pytest
import torch

from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

FIELDS = ("qbar", "kbar", "vsum", "hbar", "M", "kbar_op", "vsum_op", "hbar_op")
STATS_REL_TOL = 1e-5      # the tolerance the parity tests use for fp32 block statistics


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = C.lib()
    for seed in (11, 12):
        w = Workload("noalloc", 1, 4, (4, 16, 32), 0, 128, 64, 0.75, 0.5, "bf16", seed=seed)
        q, k, v = (x.cuda() for x in make_qkv(w))
        shape = C.shape_of(q, w.block)
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
        for f in FIELDS:
            a = getattr(got, f).float()
            b = getattr(ref, f).float()
            rel = float((a - b).norm() / b.norm().clamp_min(1e-30))
            assert rel <= STATS_REL_TOL, (seed, f, rel)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = C.lib()
    shape = C.make_shape(1, 40, 75600, 128, 128, "bf16")      # needs ~97 MB of scratch
    st = C.PisaStats()
    assert lib.pisa_precompute_noalloc(ctypes.byref(shape), 16, 16, 16, ctypes.byref(st), None) == \
        C.PISA_ERR_UNSUPPORTED
