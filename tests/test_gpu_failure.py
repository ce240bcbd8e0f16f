"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported.

The test-only hook makes the attention kernel skip its query-tile load, so the MMA warp's wait for
it can never complete.  The kernel must record PISA_DEVERR_WAIT_TIMEOUT in the workspace status
word within its (shortened) wait limit, drain its own work, free its tensor memory and return; the
next call on the same context must then run normally and match the oracle.
"""
import pytest
import torch

from oracle import pisa_oracle as O
from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import Pisa
from piecewise_approximate_attention_b200.workloads import Workload, make_qkv
from tests.parity import assert_output, compare_selection, rows_of_blocks

pytestmark = pytest.mark.gpu

SKIP_Q_LOAD = 1
WAIT_NS = 20_000_000          # 20 ms instead of the default 2 s


def test_wait_timeout_is_reported_and_context_survives():
    w = Workload("fault", 1, 1, (2, 16, 16), 0, 128, 128, 0.5, 0.5, "bf16", seed=2)
    q, k, v = make_qkv(w)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    p = Pisa(1, 1, w.seq_len, 128, w.block, w.keep_k, w.lam, "bf16", 1.0, "cuda")
    p.precompute(qd, kd, vd)
    p.route()
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    o = torch.zeros_like(qd)
    assert C.lib().pisa_testing_set_attention_fault(SKIP_Q_LOAD, WAIT_NS) == C.PISA_OK
    try:
        p.attention(qd, kd, vd, o)
        torch.cuda.synchronize()
    finally:
        assert C.lib().pisa_testing_set_attention_fault(0, 0) == C.PISA_OK
    assert p.device_error() == (C.PISA_ERR_DEVICE_TIMEOUT, C.PISA_DEVERR_WAIT_TIMEOUT)
    assert p.device_error() == (C.PISA_OK, 0)          # read clears the status word
    # the context is intact: a normal call works and is correct
    o2 = torch.empty_like(qd)
    p.attention(qd, kd, vd, o2)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    ref = O.pisa(q.double().numpy(), k.double().numpy(), v.double().numpy(), w.block, w.keep_k, w.lam)
    bad, ties = compare_selection(p.sel[0, 0].cpu().numpy(), ref["sel"][0, 0], ref["r"][0, 0], w.keep_k)
    assert not bad
    keep = ~rows_of_blocks(w.seq_len, w.block, ties)
    assert_output(o2[0, 0].double().cpu().numpy()[keep], ref["o"][0, 0][keep], "bf16", what="after timeout")


SKIP_TILE_LOAD = 2


@pytest.mark.parametrize("first_order", [True, False], ids=["first_order", "zeroth_order"])
def test_precompute_wait_timeout_is_reported_and_context_survives(first_order):
    """The pre-computation's first pass never gets the first tile of each CTA's first group: with
    10 heads x 16 groups (more groups than SMs, so several CTAs own two) every CTA's bounded wait
    runs out and it must give up all its groups, drain and return; the reduction and the second
    pass, launched as its programmatic dependents, must still end.  The status word reports the
    timeout, and the next call on the context runs normally and matches the oracle."""
    w = Workload("fault", 1, 10, (4, 64, 128), 0, 128, 128, 0.875, 0.5, "bf16", seed=4)
    q, k, v = make_qkv(w)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    lam = w.lam if first_order else 0.0
    mode = C.PISA_MODE_PISA if first_order else C.PISA_MODE_EXACT_ONLY
    p = Pisa(1, w.heads, w.seq_len, 128, w.block, w.keep_k, lam, "bf16", 1.0, "cuda", mode, first_order=first_order)
    assert C.lib().pisa_testing_set_precompute_fault(SKIP_TILE_LOAD, WAIT_NS) == C.PISA_OK
    try:
        p.precompute(qd, kd, vd)
        torch.cuda.synchronize()
    finally:
        assert C.lib().pisa_testing_set_precompute_fault(0, 0) == C.PISA_OK
    assert p.device_error() == (C.PISA_ERR_DEVICE_TIMEOUT, C.PISA_DEVERR_WAIT_TIMEOUT)
    assert p.device_error() == (C.PISA_OK, 0)
    p.precompute(qd, kd, vd)
    p.route()
    o = torch.empty_like(qd)
    p.attention(qd, kd, vd, o)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    hs = [0, 9]
    md = "pisa" if first_order else "exact_only"
    ref = O.pisa(q[:, hs].double().numpy(), k[:, hs].double().numpy(), v[:, hs].double().numpy(), w.block, w.keep_k,
                 lam, mode=md, qblocks=[0, 100, 255])
    rows = rows_of_blocks(w.seq_len, w.block, [0, 100, 255])
    for hi, h in enumerate(hs):
        bad, ties = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, hi], ref["r"][0, hi], w.keep_k)
        assert not bad
        keep = rows & ~rows_of_blocks(w.seq_len, w.block, ties)
        assert_output(o[0, h].double().cpu().numpy()[keep], ref["o"][0, hi][keep], "bf16", what=f"head {h} after timeout")


@pytest.mark.parametrize("dtype,mode", [("bf16_fp8qk", C.PISA_MODE_PISA), ("bf16", C.PISA_MODE_PER_BLOCK)])
def test_wait_timeout_in_other_paths(dtype, mode):
    """The same bounded wait in the e4m3-logit instantiation, and in the per-block mode, where the
    second kernel runs after the timed-out one on whatever the workspace holds (it waits only on
    its own copies and MMAs, so it ends too); the status is reported and the context survives."""
    w = Workload("fault", 1, 1, (2, 16, 16), 0, 128, 64, 0.5, 0.5, "bf16", seed=3)
    q, k, v = make_qkv(w)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    p = Pisa(1, 1, w.seq_len, 128, w.block, w.keep_k, w.lam, dtype, 1.0, "cuda", mode)
    p.precompute(qd, kd, vd)
    p.route()
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    o = torch.zeros_like(qd)
    assert C.lib().pisa_testing_set_attention_fault(SKIP_Q_LOAD, WAIT_NS) == C.PISA_OK
    try:
        p.attention(qd, kd, vd, o)
        torch.cuda.synchronize()
    finally:
        assert C.lib().pisa_testing_set_attention_fault(0, 0) == C.PISA_OK
    assert p.device_error() == (C.PISA_ERR_DEVICE_TIMEOUT, C.PISA_DEVERR_WAIT_TIMEOUT)
    o2 = torch.empty_like(qd)
    p.attention(qd, kd, vd, o2)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    assert torch.isfinite(o2).all()
