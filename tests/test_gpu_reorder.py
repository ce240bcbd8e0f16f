"""Token reordering (pisa_permute_rows, pisa_axis_permutation) on the GPU: bit-exact against the
oracle's gather/scatter, and PISA on reordered tokens against the oracle's pisa_reordered (needs a
B200).  Reordering follows "PAROAttention: Pattern-Aware ReOrdering for Efficient Sparse and
Quantized Attention in Visual Generation Models" (abstract), read as a permutation of the axis
order of the frames x height x width token grid."""
import numpy as np
import pytest
import torch

from oracle import pisa_oracle as O
from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import (AXIS_ORDERS, Pisa, axis_order_permutations,
                                                         choose_axis_order, reorder_tokens, restore_tokens)
from piecewise_approximate_attention_b200.workloads import Workload, make_qkv
from tests.parity import assert_output, compare_selection

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def test_axis_permutation_matches_oracle():
    for grid, extra in (((21, 45, 80), 0), ((1, 64, 64), 512), ((3, 5, 7), 3)):
        for order in AXIS_ORDERS:
            got = C.pisa_axis_permutation(grid, order, extra)
            assert np.array_equal(got, O.axis_permutation(grid, order, extra)), (grid, order)


@pytest.mark.parametrize("dtype,d,L", [(torch.bfloat16, 128, 1000), (torch.float32, 64, 777), (torch.bfloat16, 128, 75600)])
def test_permute_rows_bit_exact(dtype, d, L):
    g = torch.Generator().manual_seed(L)
    x = torch.randn((2, 3, L, d), generator=g).to(dtype).cuda()
    shared = torch.randperm(L, generator=g).to(torch.int32).cuda()
    per_head = torch.stack([torch.randperm(L, generator=g) for _ in range(6)]).to(torch.int32).cuda()
    for perm in (shared, per_head):
        y = reorder_tokens(x, perm)
        z = restore_tokens(y, perm)
        torch.cuda.synchronize()
        pn = perm.cpu().numpy()
        xn = x.float().cpu().numpy().reshape(6, L, d)
        if pn.ndim == 1:
            want = O.permute_rows(xn, pn)
        else:
            want = np.stack([O.permute_rows(xn[h], pn[h]) for h in range(6)])
        assert np.array_equal(y.float().cpu().numpy().reshape(6, L, d), want)
        assert torch.equal(z, x)


@pytest.mark.parametrize("order", ["hwt", "wht"])
def test_pisa_on_reordered_tokens(order):
    w = Workload("reorder", 1, 2, (6, 16, 16), 0, 128, 64, 0.75, 0.5, "bf16", seed=4)
    q, k, v = make_qkv(w)
    B, H, L, d = q.shape
    perm_np = O.axis_permutation(w.grid, order)
    perm = torch.from_numpy(perm_np.astype(np.int32)).cuda()
    qd, kd, vd = (reorder_tokens(x.cuda(), perm) for x in (q, k, v))
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, "bf16", 1.0, "cuda")
    o_r = torch.empty_like(qd)
    p(qd, kd, vd, o_r)
    ref = O.pisa_reordered(_np(q), _np(k), _np(v), perm_np, w.block, w.keep_k, w.lam)
    # selections live on the reordered problem: compare them there, then rerun with the oracle's
    for h in range(H):
        bad, _ = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, h], ref["r"][0, h], w.keep_k)
        assert not bad
    sel = torch.from_numpy(ref["sel"].astype(np.int32)).cuda()
    p.attention(qd, kd, vd, o_r, sel=sel)
    o = restore_tokens(o_r, perm)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    for h in range(H):
        assert_output(_np(o[0, h]), ref["o"][0, h], "bf16", what=f"{order} head {h}")


def test_choose_axis_order_picks_smallest_spread():
    w = Workload("reorder", 1, 3, (6, 16, 16), 0, 128, 64, 0.75, 0.5, "bf16", seed=8)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, "bf16", 1.0, "cuda")
    perms = axis_order_permutations(w.grid)
    chosen, idx = choose_axis_order(p, q, k, v, perms)
    torch.cuda.synchronize()
    qn, kn, vn = (_np(x) for x in (q, k, v))
    for h in range(H):
        sums = []
        for order in AXIS_ORDERS:
            pn = O.axis_permutation(w.grid, order)
            st = O.block_stats(O.permute_rows(qn[0, h], pn), O.permute_rows(kn[0, h], pn), O.permute_rows(vn[0, h], pn),
                               w.block)
            sums.append(st["M"].sum())
        sums = np.array(sums)
        pick = int(idx[h])
        # the GPU pick is the oracle's minimum, or within rounding of it
        assert sums[pick] <= sums.min() * (1 + 1e-3), (h, sums, pick)
        assert np.array_equal(chosen[h].cpu().numpy(), O.axis_permutation(w.grid, AXIS_ORDERS[pick]))
