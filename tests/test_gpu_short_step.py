"""Pre-computation and routing in one launch for short sequences (needs a B200).

pisa_precompute_route with PISA_PRECOMPUTE_ROUTE_FUSED runs, for bf16 inputs with at most 128 key
blocks, one thread-block cluster per head that does both passes of the pre-computation, the Hbar
reduction, the routing and the pairing.
It uses the same code and summation orders as the separate calls, so every array it writes must be
bit-identical to pisa_precompute followed by pisa_route; longer sequences fall back to those calls.
"""
import pytest
import torch

from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import Pisa
from piecewise_approximate_attention_b200.workloads import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu

STATS = ("qbar", "kbar", "vsum", "hbar", "M", "H", "kbar_op", "vsum_op", "hbar_op", "v_op", "vscale", "hdiff_op",
         "q8", "k8", "kbar8", "qscale", "kscale", "kbscale")

CASES = [
    # name, workload, keep_k, lambda, dtype, with_H
    ("image-dit", WORKLOADS["image-dit"], 18, 0.5, "bf16", False),
    ("L8192-keep16", WORKLOADS["sweep-L8192-s0.875"], 16, 0.5, "bf16", False),
    ("one-group", Workload("g1", 1, 3, (1, 16, 60), 0, 128, 64, 0.5, 0.5, "bf16", seed=4), 5, 0.5, "bf16", False),
    ("three-groups-ragged", Workload("g3", 2, 2, (1, 37, 64), 30, 128, 64, 0.5, 0.5, "bf16", seed=5), 7, 0.5, "bf16",
     False),
    ("block128", Workload("b128", 1, 4, (4, 24, 40), 7, 128, 128, 0.5, 0.5, "bf16", seed=6), 6, 0.5, "bf16", False),
    ("keep0", WORKLOADS["image-dit"].with_(heads=4), 0, 0.5, "bf16", False),
    ("lambda0", WORKLOADS["image-dit"].with_(heads=4), 18, 0.0, "bf16", False),
    ("all-kept", WORKLOADS["image-dit"].with_(heads=2), 72, 0.5, "bf16", False),
    ("with-H", WORKLOADS["image-dit"].with_(heads=3), 18, 0.5, "bf16", True),
    ("e4m3", WORKLOADS["image-dit"].with_(heads=3), 18, 0.5, "bf16_fp8qk", False),
    ("fallback-nb512", WORKLOADS["video-dit-small"].with_(heads=2), 64, 0.5, "bf16", False),
]


@pytest.mark.parametrize("name,w,keep_k,lam,dtype,with_H", CASES, ids=[c[0] for c in CASES])
def test_fused_equals_separate_calls(name, w, keep_k, lam, dtype, with_H):
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    mode = C.PISA_MODE_PER_BLOCK if with_H else C.PISA_MODE_PISA
    a = Pisa(B, H, L, d, w.block, keep_k, lam, dtype, 0.9, "cuda", mode)
    b = Pisa(B, H, L, d, w.block, keep_k, lam, dtype, 0.9, "cuda", mode)
    assert a.fused_short_step() == (a.nb <= 128)
    for x in (a, b):
        x.stats.buf.fill_(0x55)
        x.sel.fill_(-1)
        x.order.fill_(-1)
    sa = torch.full((B, H, a.nb, a.nb), float("nan"), device="cuda")
    sb = torch.full_like(sa, float("nan"))
    a.precompute(q, k, v)
    a.route(scores=sa)
    b.precompute_route(q, k, v, scores=sb, fused=True)
    torch.cuda.synchronize()
    assert a.device_error() == (C.PISA_OK, 0) and b.device_error() == (C.PISA_OK, 0)
    for f in STATS:
        x, y = getattr(a.stats, f), getattr(b.stats, f)
        if x is None:
            continue
        assert torch.equal(x, y), f
    assert torch.equal(a.sel, b.sel) and torch.equal(a.order, b.order) and torch.equal(sa, sb)
    oa, ob = torch.empty_like(q), torch.empty_like(q)
    a.attention(q, k, v, oa)
    b.attention(q, k, v, ob)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob)


def test_fused_step_graph_replay():
    """The captured step (one cluster launch + attention) replays to the direct result, twice."""
    w = WORKLOADS["image-dit"]
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    ref = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    o_ref = torch.empty_like(q)
    ref.precompute(q, k, v)
    ref.route()
    ref.attention(q, k, v, o_ref)
    o = torch.empty_like(q)
    g = p.capture(q, k, v, o, fused=True)
    for _ in range(2):
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
    assert p.device_error() == (C.PISA_OK, 0)
