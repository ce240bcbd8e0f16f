"""Per-block first-order variant (PISA_MODE_PER_BLOCK) on the GPU vs the fp64 oracle's
``first_order="per_block"`` (needs a B200).

The variant replaces the shared Hbar of every unselected block by the block's own H_j ("PISA:
Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 핵심 알고리즘,
first-order bullet).  Besides the output itself, the tests compare the difference between the
per-block and the global results, GPU against oracle, on inputs whose blocks have strongly
block-specific key/value covariance: there that difference is a large part of the output, so a
wrong sign, a missing block or a misplaced scale in the second kernel cannot hide inside the
output tolerance.
"""
import numpy as np
import pytest
import torch

from oracle import pisa_oracle as O
from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import Pisa
from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_block_structured, make_qkv
from tests.parity import assert_output, rows_of_blocks

pytestmark = pytest.mark.gpu

PB, GL = C.PISA_MODE_PER_BLOCK, C.PISA_MODE_PISA


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _gpu_pair(q, k, v, block, keep_k, dtype, sel_np, lam=0.5, scale=1.0):
    """GPU outputs (per-block, global) of every head with the given selections [B,H,nb,keep_k]."""
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, block, keep_k, lam, dtype, scale, "cuda", PB, True, pair=True)
    qkv = tuple(x.cuda() for x in (q, k, v))
    p.precompute(*qkv)
    p.route()
    sel = torch.from_numpy(np.ascontiguousarray(sel_np).astype(np.int32)).cuda()
    outs = []
    for mode in (PB, GL):
        o = torch.full_like(qkv[0], float("nan"))
        p.attention(*qkv, o, sel=sel, mode=mode)
        torch.cuda.synchronize()
        assert p.device_error() == (C.PISA_OK, 0)
        outs.append(_np(o))
    return p, outs[0], outs[1]


def _oracle_pair(q, k, v, block, keep_k, lam=0.5, scale=1.0, heads=None, qblocks=None):
    args = (_np(q), _np(k), _np(v), block, keep_k, lam, scale)
    pb = O.pisa(*args, first_order="per_block", heads=heads, qblocks=qblocks)
    gl = O.pisa(*args, first_order="global", heads=heads, qblocks=qblocks)
    assert np.array_equal(pb["sel"], gl["sel"])
    return pb, gl


@pytest.mark.parametrize("dtype,block", [("bf16", 64), ("bf16", 128), ("fp32", 64), ("fp32", 128)])
def test_block_structured(dtype, block):
    L, d, keep = 2000, 128, 3          # ragged last block in both block sizes
    q, k, v = make_block_structured(L, d, block, dtype, seed=3)
    pb, gl = _oracle_pair(q, k, v, block, keep)
    _, g_pb, g_gl = _gpu_pair(q, k, v, block, keep, dtype, pb["sel"])
    assert_output(g_pb[0, 0], pb["o"][0, 0], dtype, what=f"per-block {dtype} block {block}")
    assert_output(g_gl[0, 0], gl["o"][0, 0], dtype, what=f"global {dtype} block {block}")
    ref_delta = pb["o"][0, 0] - gl["o"][0, 0]
    # the inputs make the per-block term a large share of the output
    assert np.linalg.norm(ref_delta) > 0.2 * np.linalg.norm(pb["o"][0, 0])
    tol = 2e-2 if dtype == "bf16" else 1e-4
    assert _rel(g_pb[0, 0] - g_gl[0, 0], ref_delta) <= tol


def test_tiny_fp32_per_block():
    w = WORKLOADS["tiny-fp32"]
    q, k, v = make_qkv(w)
    pb, gl = _oracle_pair(q, k, v, w.block, w.keep_k, w.lam)
    p, g_pb, g_gl = _gpu_pair(q, k, v, w.block, w.keep_k, "fp32", pb["sel"], w.lam)
    for h in range(w.heads):
        assert_output(g_pb[0, h], pb["o"][0, h], "fp32", what=f"head {h} per-block")
        Href = O.block_stats(_np(q)[0, h], _np(k)[0, h], _np(v)[0, h], w.block)["H"]
        assert _rel(_np(p.stats.H[0, h]), Href) <= 1e-5
        assert _rel(g_pb[0, h] - g_gl[0, h], pb["o"][0, h] - gl["o"][0, h]) <= 1e-3


def test_operand_copy_is_scaled_difference():
    """hdiff_op = bf16(s (H_j - Hbar)) with the fp32 H and Hbar written by the same call."""
    L, d, block = 1500, 128, 64
    q, k, v = make_block_structured(L, d, block, "bf16", seed=5)
    scale = 0.75
    p = Pisa(1, 1, L, d, block, 4, 0.5, "bf16", scale, "cuda", PB, True)
    p.precompute(*(x.cuda() for x in (q, k, v)))
    torch.cuda.synchronize()
    H = p.stats.H[0, 0].double()
    Hbar = p.stats.hbar[0, 0].double()
    want = (scale * (H - Hbar)).to(torch.bfloat16).double()
    got = p.stats.hdiff_op[0, 0].double()
    # identical up to the fp32 rounding of the subtraction (one bf16 ulp at most)
    assert torch.all((got - want).abs() <= 2.0 ** -7 * want.abs() + 1e-30)
    Href = O.block_stats(_np(q)[0, 0], _np(k)[0, 0], _np(v)[0, 0], block)["H"]
    assert _rel(H.cpu().numpy(), Href) <= 1e-4


SAMPLED = [
    ("image-dit", [0, 23], None),
    ("video-dit-large", [7], [0, 1, 295, 589, 590]),
]


@pytest.mark.parametrize("name,heads,qblocks", SAMPLED, ids=[x[0] for x in SAMPLED])
def test_full_size_sampled_per_block(name, heads, qblocks):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    pb, gl = _oracle_pair(q, k, v, w.block, w.keep_k, w.lam, heads=heads, qblocks=qblocks)
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda", PB, True, pair=True)
    qkv = tuple(x.cuda() for x in (q, k, v))
    p.precompute(*qkv)
    p.route()
    sel = p.sel.clone()
    for hi, h in enumerate(heads):
        sel[0, h] = torch.from_numpy(pb["sel"][0, hi].astype(np.int32)).cuda()
    o = torch.full_like(qkv[0], float("nan"))
    p.attention(*qkv, o, sel=sel)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    rows = np.ones(L, bool) if qblocks is None else rows_of_blocks(L, w.block, qblocks)
    for hi, h in enumerate(heads):
        assert_output(_np(o[0, h])[rows], pb["o"][0, hi][rows], "bf16", what=f"{name} head {h} per-block")
    assert torch.isfinite(o).all()


def test_constant_key_blocks_reduce_to_dense():
    """Every block's keys constant: every H_j = 0, so the per-block result is dense attention."""
    L, d, block = 1024, 128, 64
    rng = np.random.default_rng(11)
    kb = rng.standard_normal((L // block, d)).astype(np.float32)
    k = np.repeat(kb, block, axis=0)
    q = (rng.standard_normal((L, d)) / np.sqrt(d)).astype(np.float32)
    v = rng.standard_normal((L, d)).astype(np.float32)
    tq, tk, tv = (torch.from_numpy(x).to(torch.bfloat16)[None, None] for x in (q, k, v))
    sel = np.tile(np.arange(2, dtype=np.int32), (1, 1, L // block, 1))
    _, g_pb, _ = _gpu_pair(tq, tk, tv, block, 2, "bf16", sel)
    dense = O.dense_attention(_np(tq)[0, 0], _np(tk)[0, 0], _np(tv)[0, 0])
    assert_output(g_pb[0, 0], dense, "bf16", what="constant keys per-block vs dense")
