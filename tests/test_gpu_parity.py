"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200).

Small cases are compared in full.  The full-size DiT shapes run on the GPU exactly as the benchmark
launches them, and are compared on sampled heads (and, for the largest, sampled query blocks) that
the oracle evaluates one by one.
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

_CACHE = {}


def _inputs(w: Workload):
    key = (w.name, w.grid, w.text_tokens, w.heads, w.batch, w.head_dim, w.dtype, w.seed)
    if key not in _CACHE:
        _CACHE.clear()
        _CACHE[key] = make_qkv(w)
    return _CACHE[key]


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _run(w: Workload, q, k, v, keep_k=None, lam=None, mode=C.PISA_MODE_PISA, with_H=False, scale=1.0):
    keep_k = w.keep_k if keep_k is None else keep_k
    lam = w.lam if lam is None else lam
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, keep_k, lam, w.dtype, scale, "cuda", mode, with_H, pair=True)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    scores = torch.empty((B, H, p.nb, p.nb), dtype=torch.float32, device="cuda")
    p.precompute(qd, kd, vd)
    p.route(scores=scores)
    p.attention(qd, kd, vd, o)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    return p, o, scores, (qd, kd, vd)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


STATS_ELEMENT_FACTOR = 10.0   # per-element bound: max |error| <= 10 tol RMS(reference)


def _check_stats(p, ref, b, hi, h, tol):
    """Block statistics of one head: relative L2 over the whole array <= tol, and element by
    element max |gpu - oracle| <= 10 tol RMS(oracle), so that a few wrong rows (a wrong M_j or
    kbar_j) cannot hide in an array-wide norm."""
    st = p.stats
    for name in ("qbar", "kbar", "vsum", "Hbar", "M"):
        g = _np(getattr(st, name.lower() if name != "M" else "M")[b, h])
        r = ref[name][b, hi]
        assert _rel(g, r) <= tol, f"{name} head {h}: rel err {_rel(g, r):.3e}"
        rms = float(np.sqrt(np.mean(r * r)))
        worst = float(np.abs(g - r).max())
        where = np.unravel_index(int(np.abs(g - r).argmax()), r.shape)
        assert worst <= STATS_ELEMENT_FACTOR * tol * rms, \
            f"{name} head {h}: element {where} off by {worst:.3e} = {worst / max(rms, 1e-300):.3e} x RMS"


def _attention_with(p, qkv, sel_np, b, h, o_like):
    """GPU attention where head (b, h) uses the given selection (the oracle's)."""
    sel = p.sel.clone()
    sel[b, h] = torch.from_numpy(sel_np.astype(np.int32)).cuda()
    o = torch.full_like(o_like, float("nan"))
    p.attention(*qkv, o, sel=sel)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_OK, 0)
    return o


def test_tiny_fp32_full():
    w = WORKLOADS["tiny-fp32"]
    q, k, v = _inputs(w)
    ref = O.pisa(_np(q), _np(k), _np(v), w.block, w.keep_k, w.lam)
    p, o, scores, qkv = _run(w, q, k, v, with_H=True)
    for h in range(w.heads):
        _check_stats(p, ref, 0, h, h, 1e-5)
        Href = np.stack([O.block_stats(_np(q)[0, h], _np(k)[0, h], _np(v)[0, h], w.block)["H"]])[0]
        Hg = _np(p.stats.H[0, h])
        assert _rel(Hg, Href) <= 1e-5
        assert np.abs(Hg - Href).max() <= STATS_ELEMENT_FACTOR * 1e-5 * np.sqrt(np.mean(Href * Href))
        bad, ties = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, h], ref["r"][0, h], w.keep_k)
        assert not bad, f"head {h}: selection rows differ beyond ties: {bad}"
        assert _rel(_np(scores[0, h]), ref["r"][0, h]) <= 1e-5
        o2 = _attention_with(p, qkv, ref["sel"][0, h], 0, h, o)
        assert_output(_np(o2[0, h]), ref["o"][0, h], "fp32", what=f"head {h} with oracle selection")
        keep = np.ones(w.seq_len, bool) & ~rows_of_blocks(w.seq_len, w.block, ties)
        assert_output(_np(o[0, h]), ref["o"][0, h], "fp32", keep, what=f"head {h} full pipeline")


FULL_SIZE = [
    ("image-dit", None, None),
    ("video-dit-small", [0, 11], None),
    ("video-dit-large", [0, 39], [0, 1, 100, 295, 296, 500, 589, 590]),
    ("sweep-L131072-s0.875", [5], [0, 777, 1024, 2047]),
    ("sweep-L8192-s0.5", [0, 15], None),
    ("sweep-L32768-s0", [3], [0, 255, 511]),
]


@pytest.mark.parametrize("name,heads,qblocks", FULL_SIZE, ids=[x[0] for x in FULL_SIZE])
def test_full_size_sampled(name, heads, qblocks):
    w = WORKLOADS[name]
    q, k, v = _inputs(w)
    p, o, scores, qkv = _run(w, q, k, v)
    hs = list(range(w.heads)) if heads is None else heads
    ref = O.pisa(_np(q[:, hs]), _np(k[:, hs]), _np(v[:, hs]), w.block, w.keep_k, w.lam, qblocks=qblocks)
    rows = np.ones(w.seq_len, bool) if qblocks is None else rows_of_blocks(w.seq_len, w.block, qblocks)
    for hi, h in enumerate(hs):
        _check_stats(p, ref, 0, hi, h, 1e-4)
        bad, ties = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, hi], ref["r"][0, hi], w.keep_k)
        assert not bad, f"head {h}: selection rows differ beyond ties: {bad[:10]}"
        o2 = _attention_with(p, qkv, ref["sel"][0, hi], 0, h, o)
        assert_output(_np(o2[0, h])[rows], ref["o"][0, hi][rows], "bf16", what=f"{name} head {h} oracle selection")
        keep = rows & ~rows_of_blocks(w.seq_len, w.block, ties)
        assert_output(_np(o[0, h])[keep], ref["o"][0, hi][keep], "bf16", what=f"{name} head {h} full pipeline")


BOUNDARY = [
    # 256 key blocks (one centroid per routing thread) and 257 (two, and a last group of one block);
    # 10 heads x 16 / 17 groups: more pre-computation groups than SMs, heads split across CTAs
    ("nb256", (4, 64, 64), 0),
    ("nb257", (4, 64, 64), 64),
]


@pytest.mark.parametrize("name,grid,text", BOUNDARY, ids=[b[0] for b in BOUNDARY])
def test_router_blocking_and_persistent_groups(name, grid, text):
    """Statistics, selections and outputs against the oracle on both sides of the router's switch
    from one to two centroids per thread, with a persistent pre-computation grid whose groups do
    not divide evenly over the CTAs."""
    w = Workload(name, 1, 10, grid, text, 128, 64, 0.875, 0.5, "bf16", seed=3)
    q, k, v = make_qkv(w)
    p, o, scores, qkv = _run(w, q, k, v)
    assert p.nb == (256 if text == 0 else 257)
    hs = [0, 5, 9]
    qblocks = [0, 127, p.nb - 1]
    ref = O.pisa(_np(q[:, hs]), _np(k[:, hs]), _np(v[:, hs]), w.block, w.keep_k, w.lam, qblocks=qblocks)
    rows = rows_of_blocks(w.seq_len, w.block, qblocks)
    for hi, h in enumerate(hs):
        _check_stats(p, ref, 0, hi, h, 1e-4)
        bad, ties = compare_selection(p.sel[0, h].cpu().numpy(), ref["sel"][0, hi], ref["r"][0, hi], w.keep_k)
        assert not bad, f"{name} head {h}: selection rows differ beyond ties: {bad[:10]}"
        o2 = _attention_with(p, qkv, ref["sel"][0, hi], 0, h, o)
        assert_output(_np(o2[0, h])[rows], ref["o"][0, hi][rows], "bf16", what=f"{name} head {h} oracle selection")


EDGE = [
    # dtype, grid, text, block, keep_k, lam, mode
    ("bf16", (10, 10, 10), 0, 64, 0, 0.5, C.PISA_MODE_PISA),
    ("bf16", (10, 10, 10), 0, 64, 16, 0.5, C.PISA_MODE_PISA),
    ("bf16", (10, 10, 10), 0, 64, 3, 0.0, C.PISA_MODE_EXACT_ONLY),
    ("bf16", (2, 5, 5), 0, 64, 1, 0.5, C.PISA_MODE_PISA),
    ("bf16", (2, 5, 5), 0, 64, 0, 0.5, C.PISA_MODE_PISA),
    ("bf16", (10, 10, 10), 0, 128, 2, 0.5, C.PISA_MODE_PISA),
    ("bf16", (1, 19, 20), 9, 64, 3, 0.5, C.PISA_MODE_PISA),
    ("bf16", (4, 16, 16), 0, 64, 5, 3.0, C.PISA_MODE_PISA),
    ("bf16", (10, 10, 10), 0, 64, 3, 0.5, C.PISA_MODE_PER_BLOCK),
    ("bf16", (10, 10, 10), 0, 64, 0, 0.5, C.PISA_MODE_PER_BLOCK),
    ("bf16", (10, 10, 10), 0, 64, 16, 0.5, C.PISA_MODE_PER_BLOCK),
    ("bf16", (2, 5, 5), 0, 64, 1, 0.5, C.PISA_MODE_PER_BLOCK),
    ("bf16", (1, 19, 20), 9, 128, 2, 0.5, C.PISA_MODE_PER_BLOCK),
    ("fp32", (10, 10, 10), 0, 64, 3, 0.5, C.PISA_MODE_PISA),
    ("fp32", (1, 19, 20), 9, 128, 2, 1.0, C.PISA_MODE_EXACT_ONLY),
    ("fp32", (2, 5, 5), 0, 64, 0, 0.5, C.PISA_MODE_PISA),
    ("fp32", (1, 19, 20), 9, 128, 2, 0.5, C.PISA_MODE_PER_BLOCK),
    ("fp32", (2, 5, 5), 0, 64, 0, 0.5, C.PISA_MODE_PER_BLOCK),
    # a single token: one block of one row (the centroid is the token, every H_j is 0)
    ("bf16", (1, 1, 1), 0, 64, 0, 0.5, C.PISA_MODE_PISA),
    ("bf16", (1, 1, 1), 0, 128, 1, 0.5, C.PISA_MODE_PISA),
    ("fp32", (1, 1, 1), 0, 64, 0, 0.5, C.PISA_MODE_PISA),
]
# the bf16 tensor-core path is built for head_dim 128 only; fp32 runs both head sizes
EDGE_CASES = [(c, hd) for c in EDGE for hd in ((64, 128) if c[0] == "fp32" else (128,))]
_MODE_NAME = {C.PISA_MODE_PISA: "pisa", C.PISA_MODE_EXACT_ONLY: "exact", C.PISA_MODE_PER_BLOCK: "perblock"}


@pytest.mark.parametrize("case,head_dim", EDGE_CASES,
                         ids=[f"{c[0]}-d{hd}-L{c[1][0]*c[1][1]*c[1][2]+c[2]}-b{c[3]}-k{c[4]}-{_MODE_NAME[c[6]]}"
                              for c, hd in EDGE_CASES])
def test_edge_cases(case, head_dim):
    dtype, grid, text, block, keep_k, lam, mode = case
    w = Workload("edge", 2, 2, grid, text, head_dim, block, 0.5, lam, dtype, seed=7)
    q, k, v = make_qkv(w)
    p, o, scores, qkv = _run(w, q, k, v, keep_k=keep_k, lam=lam, mode=mode, scale=0.9)
    md = "exact_only" if mode == C.PISA_MODE_EXACT_ONLY else "pisa"
    fo = "per_block" if mode == C.PISA_MODE_PER_BLOCK else "global"
    ref = O.pisa(_np(q), _np(k), _np(v), block, keep_k, lam, 0.9, mode=md, first_order=fo)
    for b in range(2):
        for h in range(2):
            bad, ties = compare_selection(p.sel[b, h].cpu().numpy()[:, :keep_k], ref["sel"][b, h], ref["r"][b, h],
                                          keep_k)
            assert not bad
            o2 = _attention_with(p, qkv, ref["sel"][b, h], b, h, o) if keep_k else o
            assert_output(_np(o2[b, h]), ref["o"][b, h], dtype, what=f"b{b} h{h}")


def test_constant_key_blocks_are_dense_on_gpu():
    """Keys constant inside every block: every H_j = 0 and PISA equals dense attention."""
    w = Workload("const", 1, 2, (8, 16, 16), 0, 128, 64, 0.5, 0.5, "bf16", seed=3)
    q, k, v = make_qkv(w)
    nb = w.num_blocks
    k = k.view(1, 2, nb, 64, 128)[:, :, :, :1].expand(1, 2, nb, 64, 128).reshape(1, 2, w.seq_len, 128).contiguous()
    dense = [O.dense_attention(_np(q)[0, h], _np(k)[0, h], _np(v)[0, h]) for h in range(2)]
    for keep in (0, 2, nb):
        p, o, _, _ = _run(w, q, k, v, keep_k=keep)
        for h in range(2):
            assert_output(_np(o[0, h]), dense[h], "bf16", what=f"keep {keep} head {h}")


def test_value_operand_copy_and_large_values():
    """The fp16 value operand is v / vscale with vscale a power of two; large values get a larger
    scale and the output still follows the oracle (o is linear in v)."""
    w = Workload("vscale", 1, 2, (4, 16, 16), 0, 128, 64, 0.75, 0.5, "bf16", seed=5)
    q, k, v = make_qkv(w)
    p, o, _, _ = _run(w, q, k, v)
    assert torch.equal(p.stats.vscale.cpu(), torch.ones(1, 2))
    assert torch.equal(p.stats.v_op.cpu(), v.to(torch.float16))
    big = (v.float() * 3000.0).to(torch.bfloat16)              # max |v| ~ 1.5e4 -> vscale 64
    p2, o2, _, _ = _run(w, q, k, big)
    sc = p2.stats.vscale.cpu()
    assert torch.all(sc == 64.0), sc
    ref = O.pisa(_np(q), _np(k), _np(big), w.block, w.keep_k, w.lam)
    for h in range(2):
        bad, ties = compare_selection(p2.sel[0, h].cpu().numpy(), ref["sel"][0, h], ref["r"][0, h], w.keep_k)
        assert not bad
        keep = ~rows_of_blocks(w.seq_len, w.block, ties)
        assert_output(_np(o2[0, h])[keep], ref["o"][0, h][keep], "bf16", what=f"large values head {h}")


@pytest.mark.parametrize("grid", [(21, 30, 52), (2, 59, 109)])
def test_order_is_a_permutation(grid):
    # 512 query blocks (four pairing segments of 128) and 201 (a ragged last segment of 73)
    w = WORKLOADS["video-dit-small"].with_(heads=2, grid=grid)
    q, k, v = make_qkv(w)
    p, _, _, _ = _run(w, q, k, v)
    od = p.order.cpu().numpy()
    for h in range(2):
        assert sorted(od[0, h].tolist()) == list(range(w.num_blocks))
        # pairs never straddle a segment: the two blocks of each 128-row tile lie in one segment
        tiles = od[0, h][: w.num_blocks // 2 * 2].reshape(-1, 2) // 128
        assert np.array_equal(tiles[:, 0], tiles[:, 1])


def test_deterministic():
    w = WORKLOADS["image-dit"].with_(heads=3)
    q, k, v = make_qkv(w)
    p, o1, s1, qkv = _run(w, q, k, v)
    sel1 = p.sel.clone()
    o2 = torch.empty_like(o1)
    p.precompute(*qkv)
    p.route()
    p.attention(*qkv, o2)
    torch.cuda.synchronize()
    assert torch.equal(sel1, p.sel)
    assert torch.equal(o1, o2)


def test_bad_selection_is_reported_not_faulted():
    w = WORKLOADS["image-dit"].with_(heads=1)
    q, k, v = make_qkv(w)
    p, o, _, qkv = _run(w, q, k, v)
    bad = p.sel.clone()
    bad[0, 0, 3, 0] = w.num_blocks + 5
    bad[0, 0, 7, 1] = bad[0, 0, 7, 0]
    o2 = torch.empty_like(o)
    p.attention(*qkv, o2, sel=bad)
    torch.cuda.synchronize()
    assert p.device_error() == (C.PISA_ERR_INVALID_ARG, C.PISA_DEVERR_BAD_SELECTION)
    assert p.device_error() == (C.PISA_OK, 0)


def test_graph_replay_matches_direct_calls():
    """A captured step (pre-compute, route, attention) replays to the same output as direct calls,
    and follows new inputs written into the captured buffers."""
    w = WORKLOADS["image-dit"].with_(heads=4)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    o_direct = torch.empty_like(q)
    p(q, k, v, o_direct)
    o = torch.empty_like(q)
    g = p.capture(q, k, v, o)
    o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_direct)
    q2, k2, v2 = (x.cuda() for x in make_qkv(w, seed=9))
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    g.replay()
    o2 = torch.empty_like(q)
    p(q2, k2, v2, o2)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)
    assert p.device_error() == (C.PISA_OK, 0)


def test_host_pipeline_matches_direct_calls():
    """runtime.HostPipeline (overlapped uploads, steps and downloads) gives, for every submitted
    step, the output of a direct call on the same inputs."""
    from piecewise_approximate_attention_b200.runtime import HostPipeline
    w = WORKLOADS["image-dit"].with_(heads=2)
    batches = [make_qkv(w, seed=s) for s in (0, 1, 2)]
    B, H, L, d = batches[0][0].shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    pipe = HostPipeline(p, batches[0][0])
    outs = [torch.empty_like(b[0]).pin_memory() for b in batches]
    hosts = [tuple(x.pin_memory() for x in b) for b in batches]
    for (qh, kh, vh), oh in zip(hosts, outs):
        pipe.submit(qh, kh, vh, oh)
    pipe.synchronize()
    ref = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    for (q, k, v), oh in zip(batches, outs):
        o = ref(q.cuda(), k.cuda(), v.cuda())
        torch.cuda.synchronize()
        assert torch.equal(oh, o.cpu())
    assert p.device_error() == (C.PISA_OK, 0)



def test_maximum_block_count():
    """nb = 4096, the largest supported: 262144 tokens in 64-token blocks (the router then works on
    8 query blocks per CTA and the selection bitmaps are full), sampled query blocks."""
    w = Workload("max-nb", 1, 1, (64, 64, 64), 0, 128, 64, 1.0 - 64 / 4096, 0.5, "bf16", seed=21)
    assert w.num_blocks == 4096 and w.keep_k == 64
    q, k, v = make_qkv(w)
    p, o, scores, qkv = _run(w, q, k, v)
    qblocks = [0, 1, 2047, 4094, 4095]
    ref = O.pisa(_np(q), _np(k), _np(v), w.block, w.keep_k, w.lam, qblocks=qblocks)
    _check_stats(p, ref, 0, 0, 0, 1e-4)
    bad, ties = compare_selection(p.sel[0, 0].cpu().numpy(), ref["sel"][0, 0], ref["r"][0, 0], w.keep_k)
    assert not bad, f"selection rows differ beyond ties: {bad[:10]}"
    o2 = _attention_with(p, qkv, ref["sel"][0, 0], 0, 0, o)
    rows = rows_of_blocks(w.seq_len, w.block, qblocks)
    assert_output(_np(o2[0, 0])[rows], ref["o"][0, 0][rows], "bf16", what="nb 4096, oracle selection")
