"""Seeded random shapes through the whole CUDA path against the fp64 oracle (needs a B200).

The fixed cases elsewhere pin the workloads and the edges; these draw lengths (with ragged last
blocks), block sizes, head and batch counts, sparsity, lambda, modes and input types from a fixed
seed, so that combinations no hand-written case names are also held to the same bars: block
statistics element by element, selections up to the tie rule, and the output with the oracle's
selection and through the whole pipeline.
"""
import numpy as np
import pytest
import torch

from oracle import pisa_oracle as O
from piecewise_approximate_attention_b200 import _lib as C
from piecewise_approximate_attention_b200.runtime import Pisa
from piecewise_approximate_attention_b200.workloads import Workload, make_qkv
from tests.parity import assert_output, compare_selection, rows_of_blocks

pytestmark = pytest.mark.gpu

_MODES = {"pisa": C.PISA_MODE_PISA, "exact_only": C.PISA_MODE_EXACT_ONLY, "per_block": C.PISA_MODE_PER_BLOCK}


def _cases(n=14, seed=20260301):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        dtype = "fp32" if i % 5 == 4 else "bf16"
        d = (64 if i % 10 == 4 else 128) if dtype == "fp32" else 128   # fp32 covers both head sizes
        block = int(rng.choice([64, 128]))
        L = int(rng.integers(block, 48 * block)) + (int(rng.integers(1, block)) if i % 2 else 0)
        heads = int(rng.integers(1, 4))
        batch = 2 if i % 7 == 3 else 1
        sparsity = float(rng.choice([0.5, 0.75, 0.875]))
        lam = float(rng.choice([0.0, 0.5, 2.0]))
        mode = ["pisa", "pisa", "exact_only", "per_block"][int(rng.integers(0, 4))]
        scale = float(rng.choice([1.0, 0.8]))
        out.append((i, dtype, d, block, L, heads, batch, sparsity, lam, mode, scale))
    return out


CASES = _cases()


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("case", CASES, ids=[f"c{c[0]}-{c[1]}-d{c[2]}-b{c[3]}-L{c[4]}-h{c[5]}x{c[6]}-{c[9]}"
                                             for c in CASES])
def test_random_shape_matches_oracle(case):
    i, dtype, d, block, L, heads, batch, sparsity, lam, mode, scale = case
    w = Workload(f"fuzz{i}", batch, heads, (1, 1, L), 0, d, block, sparsity, lam, dtype, seed=100 + i)
    q, k, v = make_qkv(w)
    keep = w.keep_k
    p = Pisa(batch, heads, L, d, block, keep, lam, dtype, scale, "cuda", _MODES[mode])
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    p.precompute(qd, kd, vd)
    p.route()
    p.attention(qd, kd, vd, o)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    md = "exact_only" if mode == "exact_only" else "pisa"
    fo = "per_block" if mode == "per_block" else "global"
    ref = O.pisa(_np(q), _np(k), _np(v), block, keep, lam, scale, mode=md, first_order=fo)
    tol = 1e-5 if dtype == "fp32" else 1e-4
    st = p.stats
    for b in range(batch):
        for h in range(heads):
            for name, g in (("qbar", st.qbar), ("kbar", st.kbar), ("vsum", st.vsum), ("Hbar", st.hbar), ("M", st.M)):
                gv, rv = _np(g[b, h]), ref[name][b, h]
                rms = float(np.sqrt(np.mean(rv * rv)))
                assert np.abs(gv - rv).max() <= 10 * tol * max(rms, 1e-30), f"{name} b{b} h{h}"
            bad, ties = compare_selection(p.sel[b, h].cpu().numpy(), ref["sel"][b, h], ref["r"][b, h], keep)
            assert not bad, f"b{b} h{h}: selection rows differ beyond ties: {bad[:8]}"
            sel = p.sel.clone()
            sel[b, h] = torch.from_numpy(ref["sel"][b, h].astype(np.int32)).cuda()
            o2 = torch.full_like(qd, float("nan"))
            p.attention(qd, kd, vd, o2, sel=sel)
            torch.cuda.synchronize()
            assert p.device_error() == (C.PISA_OK, 0)
            assert_output(_np(o2[b, h]), ref["o"][b, h], dtype, what=f"b{b} h{h} oracle selection")
            rows = ~rows_of_blocks(L, block, ties)
            assert_output(_np(o[b, h])[rows], ref["o"][b, h][rows], dtype, what=f"b{b} h{h} full pipeline")
