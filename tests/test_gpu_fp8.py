"""e4m3 logits for the exact stage (dtype PISA_BF16_FP8QK) on the GPU vs the oracle's pisa_fp8
(needs a B200).

The quantized copies are integer work and must match bit for bit where both sides quantize the
same float32 numbers (q and k, read from the same bf16 inputs); the centroids are quantized from
each side's own kbar (float32 on the GPU, float64 in the oracle), so their codes may differ by one
step at a rounding boundary.  The attention output is held to the bf16 budget against the oracle
evaluated on the same e4m3 values: quantization itself is part of what both sides compute.
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


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _codes(u8):
    """e4m3 bytes -> their values (float64)."""
    return u8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _pisa(w, q, k, v, keep_k, mode=C.PISA_MODE_PISA, scale=1.0):
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, keep_k, w.lam, "bf16_fp8qk", scale, "cuda", mode)
    qkv = tuple(x.cuda() for x in (q, k, v))
    p.precompute(*qkv)
    p.route()
    torch.cuda.synchronize()
    return p, qkv


def test_quantized_copies_match_oracle():
    w = Workload("f8", 1, 2, (5, 10, 20), 24, 128, 64, 0.75, 0.5, "bf16", seed=12)
    q, k, v = make_qkv(w)
    p, _ = _pisa(w, q, k, v, w.keep_k)
    st = p.stats
    L, nb = w.seq_len, w.num_blocks
    for h in range(w.heads):
        qn, kn, vn = _np(q[0, h]), _np(k[0, h]), _np(v[0, h])
        qd, qs = O.quantize_groups(qn, np.arange(L))
        assert np.array_equal(st.qscale[0, h].cpu().numpy(), qs)
        assert np.array_equal(_codes(st.q8[0, h]) * qs[:, None].astype(np.float64), qd)
        kd, ks = O.quantize_groups(kn, np.arange(L) // w.block)
        assert np.array_equal(st.kscale[0, h].cpu().numpy(), ks)
        assert np.array_equal(_codes(st.k8[0, h]) * ks[np.arange(L) // w.block][:, None].astype(np.float64), kd)
        kbar = O.block_stats(qn, kn, vn, w.block)["kbar"]
        kbd, kbs = O.quantize_groups(kbar, np.arange(nb) // 128)
        gs = st.kbscale[0, h].cpu().numpy().astype(np.float64)
        assert np.allclose(gs, kbs, rtol=1e-6)
        got = _codes(st.kbar8[0, h]) * gs[np.arange(nb) // 128][:, None]
        # one e4m3 step at most (2^-3 relative for normal codes, 2^-9 * scale for subnormal ones)
        assert np.all(np.abs(got - kbd) <= 2.0 ** -3 * np.abs(kbd) + 2.0 ** -9 * gs[0] + 1e-12)


CASES = [
    # grid, text, block, keep_k, mode
    ((10, 10, 10), 0, 64, 3, C.PISA_MODE_PISA),
    ((10, 10, 10), 0, 64, 0, C.PISA_MODE_PISA),
    ((10, 10, 10), 0, 64, 16, C.PISA_MODE_PISA),
    ((10, 10, 10), 0, 64, 3, C.PISA_MODE_EXACT_ONLY),
    ((1, 19, 20), 9, 128, 2, C.PISA_MODE_PISA),
    ((2, 5, 5), 0, 64, 1, C.PISA_MODE_PISA),
    ((4, 16, 16), 0, 64, 5, C.PISA_MODE_PISA),
]


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0][0]*c[0][1]*c[0][2]+c[1]}-b{c[2]}-k{c[3]}-m{c[4]}" for c in CASES])
def test_fp8_attention_parity(case):
    grid, text, block, keep, mode = case
    w = Workload("f8", 2, 2, grid, text, 128, block, 0.5, 0.5, "bf16", seed=7)
    q, k, v = make_qkv(w)
    p, qkv = _pisa(w, q, k, v, keep, mode, scale=0.9)
    md = "exact_only" if mode == C.PISA_MODE_EXACT_ONLY else "pisa"
    ref = O.pisa_fp8(_np(q), _np(k), _np(v), block, keep, w.lam, 0.9, mode=md)
    sel = p.sel.clone()
    for b in range(2):
        for h in range(2):
            if keep:
                bad, _ = compare_selection(p.sel[b, h].cpu().numpy()[:, :keep], ref["sel"][b, h], ref["r"][b, h], keep)
                assert not bad
                sel[b, h, :, :keep] = torch.from_numpy(ref["sel"][b, h].astype(np.int32)).cuda()
    o = torch.full_like(qkv[0], float("nan"))
    p.attention(*qkv, o, sel=sel)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    for b in range(2):
        for h in range(2):
            assert_output(_np(o[b, h]), ref["o"][b, h], "bf16", what=f"b{b} h{h}")


SAMPLED = [("image-dit", [0, 23], None), ("video-dit-large", [5], [0, 1, 300, 589, 590])]


@pytest.mark.parametrize("name,heads,qblocks", SAMPLED, ids=[x[0] for x in SAMPLED])
def test_fp8_full_size_sampled(name, heads, qblocks):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    p, qkv = _pisa(w, q, k, v, w.keep_k)
    ref = O.pisa_fp8(_np(q[:, heads]), _np(k[:, heads]), _np(v[:, heads]), w.block, w.keep_k, w.lam,
                     qblocks=qblocks)
    sel = p.sel.clone()
    for hi, h in enumerate(heads):
        bad, _ = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, hi], ref["r"][0, hi], w.keep_k)
        assert not bad
        sel[0, h] = torch.from_numpy(ref["sel"][0, hi].astype(np.int32)).cuda()
    o = torch.full_like(qkv[0], float("nan"))
    p.attention(*qkv, o, sel=sel)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    rows = np.ones(w.seq_len, bool) if qblocks is None else rows_of_blocks(w.seq_len, w.block, qblocks)
    for hi, h in enumerate(heads):
        assert_output(_np(o[0, h])[rows], ref["o"][0, hi][rows], "bf16", what=f"{name} head {h}")
    assert torch.isfinite(o).all()
