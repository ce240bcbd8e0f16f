"""The zeroth-order pre-computation and the keep-or-drop pipeline it serves (needs a B200).

pisa_precompute_zeroth_order writes the statistics that routing without the covariance term and
the keep-or-drop mode read; they must equal pisa_precompute's bit for bit (same kernels for the
block sums, the fp16 value operand written in the first pass and rewritten when the head's value
scale is not 1).  The pipeline zeroth-order pre-compute -> lambda = 0 routing -> PISA_MODE_EXACT_ONLY
is checked against the oracle's keep-or-drop mode.
"""
import numpy as np
import pytest
import torch

from oracle import pisa_oracle as O
from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import Pisa
from piecewise_approximate_attention_b200.workloads import WORKLOADS, Workload, make_qkv
from tests.parity import assert_output, compare_selection, rows_of_blocks

pytestmark = pytest.mark.gpu

ZEROTH = ("qbar", "kbar", "vsum", "kbar_op", "vsum_op", "v_op", "vscale", "q8", "k8", "kbar8", "qscale", "kscale",
          "kbscale")


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("dtype,head_dim,block,vmul", [
    ("bf16", 128, 64, 1.0), ("bf16", 128, 128, 1.0), ("bf16", 128, 64, 3000.0), ("bf16", 128, 128, 1e6),
    ("fp32", 64, 64, 1.0), ("fp32", 128, 128, 1.0), ("bf16_fp8qk", 128, 64, 1.0)])
def test_zeroth_order_statistics_equal_full_precompute(dtype, head_dim, block, vmul):
    # 2 heads x 1300 tokens (short last block); vmul > 256 makes the value scale > 1 (the rewrite)
    w = Workload("zeroth", 1, 2, (1, 26, 50), 0, head_dim, block, 0.75, 0.5, "fp32" if dtype == "fp32" else "bf16",
                 seed=31)
    q, k, v = (x.cuda() for x in make_qkv(w))
    if vmul != 1.0:
        v = (v.float() * vmul).to(v.dtype)
    shape = C.make_shape(1, 2, w.seq_len, head_dim, block, dtype)
    full = C.alloc_stats(shape, "cuda")
    zero = C.alloc_stats(shape, "cuda")
    zero.buf.fill_(0x7F)
    ws = C.alloc_workspace(shape, "cuda")
    C.pisa_precompute(shape, q, k, v, full, ws)
    C.pisa_precompute_zeroth_order(shape, q, k, v, zero, ws)
    torch.cuda.synchronize()
    assert C.pisa_read_device_error(ws) == (C.PISA_OK, 0)
    compared = 0
    for f in ZEROTH:
        a, b = getattr(zero, f), getattr(full, f)
        if b is None:
            continue
        assert torch.equal(a, b), f
        compared += 1
    assert compared >= (13 if dtype == "bf16_fp8qk" else 7 if dtype == "bf16" else 3)
    if dtype == "bf16" and vmul > 256:
        assert float(full.vscale.min()) > 1.0


@pytest.mark.parametrize("name,heads,qblocks", [
    ("image-dit", [0, 23], None),
    ("video-dit-large", [7], [0, 1, 300, 590]),
    ("sweep-L8192-s0.875", [2], None),
])
def test_keep_or_drop_pipeline_matches_oracle(name, heads, qblocks):
    """zeroth-order pre-compute -> lambda = 0 route -> PISA_MODE_EXACT_ONLY, as the bench's
    exact-only arm runs it, against the oracle's keep-or-drop mode on sampled heads."""
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, heads=heads)
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, 0.0, w.dtype, 1.0, "cuda", C.PISA_MODE_EXACT_ONLY, first_order=False)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    # M is never written by the zeroth-order pre-computation: poison it, routing must not read it
    p.stats.M.fill_(float("nan"))
    o = torch.full_like(qd, float("nan"))
    scores = torch.empty((B, H, p.nb, p.nb), dtype=torch.float32, device="cuda")
    p.precompute(qd, kd, vd)
    p.route(scores=scores)
    p.attention(qd, kd, vd, o)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    assert bool(torch.isfinite(scores).all())
    ref = O.pisa(_np(q), _np(k), _np(v), w.block, w.keep_k, 0.0, mode="exact_only", qblocks=qblocks)
    rows = np.ones(L, bool) if qblocks is None else rows_of_blocks(L, w.block, qblocks)
    for h in range(H):
        bad, ties = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, h], ref["r"][0, h], w.keep_k)
        assert not bad, f"{name} head {h}: selection rows differ beyond ties: {bad[:10]}"
        keep = rows & ~rows_of_blocks(L, w.block, ties)
        assert_output(_np(o[0, h])[keep], ref["o"][0, h][keep], "bf16", what=f"{name} head {h} keep-or-drop")


def test_lambda_zero_route_ignores_M():
    """With lambda = 0 the selection does not depend on what M holds."""
    w = WORKLOADS["image-dit"].with_(heads=2)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, 0.0, w.dtype, 1.0, "cuda")
    p.precompute(q, k, v)
    p.route()
    sel1 = p.sel.clone()
    p.stats.M.fill_(float("nan"))
    p.route()
    torch.cuda.synchronize()
    assert torch.equal(sel1, p.sel)
