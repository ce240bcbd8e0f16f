"""Pins for the fp64 oracle: checks against facts fixed outside the oracle itself.

Each pin returns (ok, detail).  Sources of truth, none of which re-types the oracle's formulas:
  * a library routine (torch scaled_dot_product_attention in float64, numpy.cov, numpy.linalg.norm)
    for the special cases where PISA reduces to it (all blocks selected, block size 1, blocks of
    constant keys, keep-or-drop with a block mask);
  * invariances the method must have (value shift and scale, permutation inside a block);
  * the order of the Taylor error as the key spread eps -> 0 (second order when every block has the
    same first-order matrix, first order in general, second order with per-block matrices);
  * a literal token-by-token evaluator of the Taylor expansion (brute force, L <= 256);
  * hand-built routing cases whose selections follow from the combination rule in closed form.
The method is "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers"
(§2 방법론: numerator equation, covariance-aware routing).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import pisa_oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa(q, k, v, scale, mask=None):
    import torch
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m, scale=scale)[0, 0].numpy()


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _run(q, k, v, block, keep_k, lam, scale=1.0, **kw):
    res = O.pisa(q[None, None], k[None, None], v[None, None], block, keep_k, lam, scale, **kw)
    return res["o"][0, 0], res


def _qkv(seed, L, d, dv=None, spread=1.0):
    r = _rng(seed)
    dv = d if dv is None else dv
    return r.standard_normal((L, d)) * spread, r.standard_normal((L, d)) * spread, r.standard_normal((L, dv))


# ---------------------------------------------------------------------------------------------
# Output pins
# ---------------------------------------------------------------------------------------------
def pin_all_selected_is_dense():
    """keep_k = nb: every block exact -> softmax attention (torch SDPA, fp64)."""
    q, k, v = _qkv(1, 200, 8)
    worst = 0.0
    for block in (16, 24, 64):
        nb = O.num_blocks(200, block)
        for scale in (1.0, 0.6):
            o, _ = _run(q, k, v, block, nb, 0.5, scale)
            worst = max(worst, _rel(o, _sdpa(q, k, v, scale)))
    return worst < 1e-12, f"max rel err {worst:.3e}"


def pin_block_one_is_dense():
    """block = 1: kbar = k, every H_j = 0 -> dense attention for every keep_k and lambda."""
    q, k, v = _qkv(2, 48, 6)
    worst = 0.0
    for keep in (0, 1, 7, 48):
        for lam in (0.0, 0.5):
            o, _ = _run(q, k, v, 1, keep, lam, 0.8)
            worst = max(worst, _rel(o, _sdpa(q, k, v, 0.8)))
    return worst < 1e-12, f"max rel err {worst:.3e}"


def pin_constant_key_blocks_are_dense():
    """Keys constant inside every block (ragged tail included): the expansion is exact."""
    r = _rng(3)
    L, d, block = 70, 5, 16
    nb = O.num_blocks(L, block)
    centers = r.standard_normal((nb, d))
    k = np.concatenate([np.repeat(centers[j][None], min(block, L - j * block), 0) for j in range(nb)])
    q = r.standard_normal((L, d))
    v = r.standard_normal((L, d)) + 0.3
    worst = 0.0
    for keep in (0, 1, 3):
        for lam in (0.0, 0.5, 1e3):
            o, _ = _run(q, k, v, block, keep, lam, 0.9)
            worst = max(worst, _rel(o, _sdpa(q, k, v, 0.9)))
    return worst < 1e-12, f"max rel err {worst:.3e}"


def pin_exact_only_is_masked_sdpa():
    """Keep-or-drop mode equals SDPA with a boolean block mask built from the same selection."""
    q, k, v = _qkv(4, 100, 6)
    block, keep = 16, 3
    o, res = _run(q, k, v, block, keep, 0.5, 1.0, mode="exact_only")
    sel = res["sel"][0, 0]
    mask = np.zeros((100, 100), dtype=bool)
    for i in range(sel.shape[0]):
        for j in sel[i]:
            mask[i * block:(i + 1) * block, j * block:(j + 1) * block] = True
    err = _rel(o, _sdpa(q, k, v, 1.0, mask))
    return err < 1e-12, f"rel err {err:.3e}"


def pin_brute_force_matches():
    """Blocked evaluator == literal per-token Taylor evaluator (d != dv, ragged tail, both orders)."""
    worst = 0.0
    for seed, L, block, keep, scale in ((5, 40, 8, 2, 0.7), (6, 37, 16, 1, 1.3), (7, 24, 8, 0, 0.5)):
        q, k, v = _qkv(seed, L, 4, 3)
        for fo in ("global", "per_block"):
            o, res = _run(q, k, v, block, keep, 0.5, scale, first_order=fo)
            bf = O.brute_force_head(q, k, v, block, res["sel"][0, 0], scale, fo)
            worst = max(worst, _rel(o, bf))
    return worst < 1e-12, f"max rel err {worst:.3e}"


def pin_value_shift_equivariance():
    """o(v + c) = o(v) + c: needs D = exact mass + sum cnt_j alpha_j and a centred H_j."""
    q, k, v = _qkv(8, 90, 6)
    c = _rng(9).standard_normal(6) * 3.0
    o1, _ = _run(q, k, v, 16, 2, 0.5, 0.8)
    o2, _ = _run(q, k, v + c[None], 16, 2, 0.5, 0.8)
    err = float(np.abs(o2 - (o1 + c[None])).max())
    return err < 1e-11, f"max abs err {err:.3e}"


def pin_value_scale_linearity():
    """o(a v) = a o(v)."""
    q, k, v = _qkv(10, 90, 6)
    o1, _ = _run(q, k, v, 16, 2, 0.5)
    o2, _ = _run(q, k, -2.5 * v, 16, 2, 0.5)
    err = _rel(o2, -2.5 * o1)
    return err < 1e-12, f"rel err {err:.3e}"


def pin_in_block_permutation():
    """Permuting tokens inside each block permutes the output rows the same way, nothing else."""
    q, k, v = _qkv(11, 75, 5)
    block = 16
    r = _rng(12)
    perm = np.concatenate([s + r.permutation(e - s) for s, e in O.block_bounds(75, block)])
    o1, _ = _run(q, k, v, block, 2, 0.5)
    o2, _ = _run(q[perm], k[perm], v[perm], block, 2, 0.5)
    err = _rel(o2, o1[perm])
    return err < 1e-12, f"rel err {err:.3e}"


def _taylor_errors(shared_structure: bool, first_order: str, scale=0.5, seed=13):
    r = _rng(seed)
    L, block, d = 64, 8, 4
    nb = L // block
    centers = r.standard_normal((nb, d))
    delta = r.standard_normal((nb, block, d))
    if shared_structure:
        delta[:] = delta[0]
    delta -= delta.mean(axis=1, keepdims=True)              # block mean stays at its center
    V0 = r.standard_normal((block, d))
    v = np.concatenate([V0 if shared_structure else r.standard_normal((block, d)) for _ in range(nb)])
    q = r.standard_normal((L, d))
    errs = []
    for eps in (0.08, 0.04, 0.02):
        k = (centers[:, None, :] + eps * delta).reshape(L, d)
        o, _ = _run(q, k, v, block, 0, 0.5, scale, first_order=first_order)
        errs.append(float(np.abs(o - _sdpa(q, k, v, scale)).max()))
    return errs


def pin_second_order_when_blocks_share_structure():
    """keep_k = 0 and every H_j equal (= Hbar): error vs dense falls as eps^2 (halving eps -> /4)."""
    e = _taylor_errors(True, "global")
    ratios = [e[0] / e[1], e[1] / e[2]]
    return min(ratios) > 3.3, f"errors {e}, ratios {ratios}"


def pin_first_order_in_general():
    """Distinct H_j: global Hbar leaves an O(eps) error (ratio ~2), per-block H_j an O(eps^2) one."""
    g = _taylor_errors(False, "global")
    p = _taylor_errors(False, "per_block")
    rg = [g[0] / g[1], g[1] / g[2]]
    rp = [p[0] / p[1], p[1] / p[2]]
    ok = all(1.6 < x < 2.6 for x in rg) and min(rp) > 3.3 and p[2] < g[2]
    return ok, f"global ratios {rg}, per-block ratios {rp}"


# ---------------------------------------------------------------------------------------------
# Statistics pins
# ---------------------------------------------------------------------------------------------
def pin_block_means_and_sums():
    """qbar, kbar are block means and vsum block sums (numpy mean/sum), ragged tail by its count."""
    q, k, v = _qkv(14, 70, 5)
    st = O.block_stats(q, k, v, 16)
    worst = 0.0
    for j, (s, e) in enumerate(O.block_bounds(70, 16)):
        worst = max(worst, np.abs(st["qbar"][j] - np.mean(q[s:e], 0)).max(),
                    np.abs(st["kbar"][j] - np.mean(k[s:e], 0)).max(),
                    np.abs(st["vsum"][j] - np.sum(v[s:e], 0)).max())
        if st["cnt"][j] != e - s:
            return False, "bad cnt"
    return worst < 1e-13, f"max abs err {worst:.3e}"


def pin_first_order_matrix_is_cross_covariance():
    """H_j = cnt_j * biased cross-covariance(k, v) of the block (numpy.cov)."""
    q, k, v = _qkv(15, 70, 5, 3)
    st = O.block_stats(q, k, v, 16)
    worst = 0.0
    for j, (s, e) in enumerate(O.block_bounds(70, 16)):
        C = np.cov(k[s:e].T, v[s:e].T, bias=True)[:5, 5:]
        worst = max(worst, np.abs(st["H"][j] - (e - s) * C).max())
    return worst < 1e-12, f"max abs err {worst:.3e}"


def pin_global_statistic_closed_form():
    """One block with spread, all others constant: Hbar = H_0 / nb and M_j = ||H_0||_F / nb (j > 0)."""
    r = _rng(16)
    L, block, d = 64, 16, 4
    nb = L // block
    k = np.repeat(r.standard_normal((nb, d)), block, axis=0)
    k[:block] += r.standard_normal((block, d))
    q = r.standard_normal((L, d))
    v = r.standard_normal((L, d))
    st = O.block_stats(q, k, v, block)
    H0 = (k[:block] - k[:block].mean(0)).T @ v[:block]
    e1 = np.abs(st["Hbar"] - H0 / nb).max()
    e2 = np.abs(st["M"][1:] - np.linalg.norm(H0, "fro") / nb).max()
    e3 = abs(st["M"][0] - np.linalg.norm(H0 * (1 - 1 / nb), "fro"))
    worst = max(e1, e2, e3)
    return worst < 1e-12, f"max abs err {worst:.3e}"


def pin_cov_norm():
    """Frobenius M_j matches numpy.linalg.norm('fro'); the spectral diagnostic never exceeds it."""
    q, k, v = _qkv(17, 96, 6)
    st = O.block_stats(q, k, v, 16)
    sp = O.block_stats(q, k, v, 16, norm="spectral")
    ref = np.array([np.linalg.norm(st["H"][j] - st["Hbar"], "fro") for j in range(6)])
    e = np.abs(st["M"] - ref).max()
    ok = e < 1e-12 and np.all(sp["M"] <= st["M"] + 1e-12) and np.all(sp["M"] > 0)
    return ok, f"max abs err {e:.3e}"


# ---------------------------------------------------------------------------------------------
# Routing pins
# ---------------------------------------------------------------------------------------------
def _stats(qbar, kbar, cnt, M):
    return dict(qbar=np.asarray(qbar, float), kbar=np.asarray(kbar, float),
                cnt=np.asarray(cnt, dtype=np.int64), M=np.asarray(M, float))


def pin_route_combination_rule():
    """P = [0.6, 0.4], M = [0.4, 1.6] (normalised [0.2, 0.8]): lambda 0.5 picks block 1, 0.2 block 0."""
    st = _stats([[math.log(1.5)]], [[1.0], [0.0]], [8, 8], [0.4, 1.6])
    r1 = O.route_scores(st, 0.5)
    r2 = O.route_scores(st, 0.2)
    ok = (np.allclose(r1, [[0.7, 0.8]], atol=1e-14) and np.allclose(r2, [[0.64, 0.56]], atol=1e-14)
          and O.route_select(r1, 1)[0, 0] == 1 and O.route_select(r2, 1)[0, 0] == 0)
    return ok, f"{r1} {r2}"


def pin_route_count_weighting():
    """A ragged 1-token block loses to a full 8-token block whose centroid score is lower by < ln 8."""
    st = _stats([[1.0]], [[1.0], [0.0], [2.0]], [8, 8, 1], [0.0, 0.0, 0.0])
    # scores 1, 0, 2; cnt-weighted log-mass 1+ln8, ln8, 2 -> block 0 first, then 1, then 2
    sel = O.route_select(O.route_scores(st, 0.0), 2)
    return list(sel[0]) == [0, 1], f"sel {sel}"


def pin_route_lambda_zero_is_pooled_topk():
    """lambda = 0: S_i = top-k of s q̄_i.k̄_j + ln cnt_j (softmax is monotone), checked by argsort."""
    q, k, v = _qkv(18, 150, 6)
    st = O.block_stats(q, k, v, 16)
    sel = O.route_select(O.route_scores(st, 0.0, 0.7), 4)
    logit = 0.7 * st["qbar"] @ st["kbar"].T + np.log(st["cnt"])[None]
    ref = np.sort(np.argsort(-logit, axis=1, kind="stable")[:, :4], axis=1)
    return np.array_equal(sel, ref), "mismatch" if not np.array_equal(sel, ref) else "ok"


def pin_route_large_lambda_is_cov_topk():
    """lambda -> inf: every query block selects the keep_k blocks of largest M_j."""
    q, k, v = _qkv(19, 150, 6)
    st = O.block_stats(q, k, v, 16)
    sel = O.route_select(O.route_scores(st, 1e9), 3)
    ref = np.sort(np.argsort(-st["M"], kind="stable")[:3])
    return bool(np.all(sel == ref[None])), f"sel {sel[0]} ref {ref}"


def pin_route_edges():
    """keep_k = nb selects everything; keep_k = 0 nothing; exact ties go to the lower index."""
    q, k, v = _qkv(20, 64, 4)
    st = O.block_stats(q, k, v, 16)
    all_sel = O.route_select(O.route_scores(st, 0.5), 4)
    none_sel = O.route_select(O.route_scores(st, 0.5), 0)
    tie = _stats([[1.0]], [[0.5], [0.5], [0.5], [0.1]], [4, 4, 4, 4], [1.0, 1.0, 1.0, 1.0])
    tsel = O.route_select(O.route_scores(tie, 0.5), 2)
    ok = (np.array_equal(all_sel, np.tile(np.arange(4), (4, 1))) and none_sel.shape == (4, 0)
          and list(tsel[0]) == [0, 1])
    return ok, f"tie sel {tsel}"


# ---------------------------------------------------------------------------------------------
# Token reordering pins ("PAROAttention: Pattern-Aware ReOrdering ...", abstract)
# ---------------------------------------------------------------------------------------------
def pin_axis_permutation_by_hand():
    """A 2 x 2 x 3 grid listed as (h, w, t): t runs fastest, so positions alternate between the two
    frames, 6 raster indices apart; identity for (t, h, w); extra tokens stay at the end."""
    hwt = O.axis_permutation((2, 2, 3), "hwt")
    want = [0, 6, 1, 7, 2, 8, 3, 9, 4, 10, 5, 11]          # written out from (h, w, t) = (0,0,0), (0,0,1), ...
    ident = O.axis_permutation((2, 2, 3), "thw", extra_tokens=2)
    wht = O.axis_permutation((1, 2, 2), "wht")
    # gather semantics: row i of the output is row perm[i] of the input (rows labelled by index)
    rows = O.permute_rows(np.arange(12.0)[:, None], hwt)[:, 0]
    ok = (list(hwt) == want and list(ident) == list(range(14)) and list(wht) == [0, 2, 1, 3]
          and list(rows) == want)
    return ok, f"hwt {list(hwt)} rows {list(rows)}"


def pin_axis_permutation_coordinates():
    """Every order is a permutation, and consecutive positions step by one along the fastest axis."""
    T, Hg, W = 3, 4, 5
    ok = True
    for order in ("thw", "twh", "htw", "hwt", "wth", "wht"):
        perm = O.axis_permutation((T, Hg, W), order)
        ok &= sorted(perm.tolist()) == list(range(T * Hg * W))
        t, h, w = perm // (Hg * W), (perm // W) % Hg, perm % W
        coord = {"t": t, "h": h, "w": w}
        fast = coord[order[2]]
        n_fast = {"t": T, "h": Hg, "w": W}[order[2]]
        ok &= bool(np.all(fast == np.arange(T * Hg * W) % n_fast))
    return ok, ""


def pin_permute_rows_inverse_and_dense_equivariance():
    """Scatter undoes gather; dense attention commutes with reordering the tokens (a property of
    softmax attention, checked against torch SDPA): SDPA(Pq, Pk, Pv) = P SDPA(q, k, v)."""
    q, k, v = _qkv(31, 60, 8)
    perm = O.axis_permutation((3, 4, 5), "wht")
    back = O.permute_rows(O.permute_rows(v, perm), perm, inverse=True)
    lhs = _sdpa(O.permute_rows(q, perm), O.permute_rows(k, perm), O.permute_rows(v, perm), 0.7)
    rhs = O.permute_rows(_sdpa(q, k, v, 0.7), perm)
    e = _rel(lhs, rhs)
    return np.array_equal(back, v) and e < 1e-12, f"rel {e:.2e}"


def pin_reordered_pisa_all_selected_is_dense():
    """PISA on reordered tokens with every block selected, put back in order = dense attention."""
    q, k, v = _qkv(32, 60, 8)
    perm = O.axis_permutation((3, 4, 5), "hwt")
    r = O.pisa_reordered(q[None, None], k[None, None], v[None, None], perm, 16, 4, 0.5, 0.9)
    e = _rel(r["o"][0, 0], _sdpa(q, k, v, 0.9))
    return e < 1e-12, f"rel {e:.2e}"


# ---------------------------------------------------------------------------------------------
# e4m3 logits (reading for the low-bit exact stage)
# ---------------------------------------------------------------------------------------------
def pin_e4m3_by_hand():
    """e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals down to 2^-9, largest
    finite 448) rounding to nearest, ties to even, worked out by hand from that definition."""
    x = np.array([1.0, 1.0625, 1.1875, 0.1, 2.0 ** -9, 3 * 2.0 ** -10, 448.0, 447.9999, 240.0, 250.0, -3.3])
    want = [1.0, 1.0, 1.25, 0.1015625, 2.0 ** -9, 2.0 ** -8, 448.0, 448.0, 240.0, 256.0, -3.25]
    got = O.e4m3(x)
    return bool(np.array_equal(got, want)), f"{got}"


def pin_quantize_groups_bounds():
    """Each group's largest |x| maps to the code 448; every value is within half a unit in the last
    place (2^-4 relative, or 2^-10 * scale for subnormal codes)."""
    x = _rng(40).standard_normal((12, 16)) * np.linspace(0.01, 5, 12)[:, None]
    groups = np.arange(12) // 4
    d, sc = O.quantize_groups(x, groups)
    ok = True
    for g in range(3):
        rows = groups == g
        big = np.abs(x[rows]).max()
        ok &= abs(np.abs(d[rows]).max() - 448.0 * float(sc[g])) <= 1e-12 * big
        ok &= abs(float(sc[g]) - np.float32(np.float32(big) / np.float32(448.0))) == 0.0
        err = np.abs(d[rows] - x[rows])
        ok &= bool(np.all(err <= 2.0 ** -4 * np.abs(x[rows]) + 2.0 ** -10 * float(sc[g]) + 1e-12))
    return bool(ok), ""


def _representable(r, n, d, scale_of_row, big_every=1):
    """Rows of e4m3 codes times a per-row factor; every `big_every`-th row holds the code +-448
    once, the others only smaller codes (so a group of big_every rows has its maximum in one row)."""
    codes = np.array([1.0, 0.5, 2.0, 3.25, 96.0, 0.1015625, 13.0, 40.0, 1.75, 0.375])
    x = r.choice(np.concatenate([codes, -codes]), size=(n, d))
    big = np.arange(n) % big_every == 0
    x[big, 0] = 448.0 * np.where(r.random(int(big.sum())) < 0.5, 1.0, -1.0)
    return x * scale_of_row[:, None]


def pin_fp8_exact_on_representable_inputs():
    """q rows that are e4m3 codes times a row factor and key blocks that are codes times a block
    factor quantize exactly (per-row q scales, per-block k scales): with every block selected the
    e4m3-logit attention equals softmax attention (torch SDPA)."""
    r = _rng(41)
    L, d, block = 64, 8, 16
    q = _representable(r, L, d, 0.003 * (1.0 + r.random(L)))
    k = _representable(r, L, d, np.repeat(0.002 * (1.0 + r.random(L // block)), block), big_every=block)
    v = r.standard_normal((L, d))
    o = O.pisa_fp8(q[None, None], k[None, None], v[None, None], block, L // block, 0.5, 0.8)["o"][0, 0]
    e = _rel(o, _sdpa(q, k, v, 0.8))
    return e < 1e-6, f"rel {e:.2e}"


def pin_fp8_constant_key_blocks_are_dense():
    """Blocks of one constant, exactly representable key (the same factor for every block, so the
    centroid tile quantizes exactly too): any keep_k gives softmax attention."""
    r = _rng(42)
    L, d, block = 64, 8, 16
    q = _representable(r, L, d, 0.003 * (1.0 + r.random(L)))
    c = _representable(r, L // block, d, np.full(L // block, 2.0 ** -8))
    k = np.repeat(c, block, axis=0)
    v = r.standard_normal((L, d))
    dense = _sdpa(q, k, v, 0.8)
    worst = 0.0
    for keep in (0, 1, 4):
        o = O.pisa_fp8(q[None, None], k[None, None], v[None, None], block, keep, 0.5, 0.8)["o"][0, 0]
        worst = max(worst, _rel(o, dense))
    return worst < 1e-6, f"rel {worst:.2e}"


def pin_fp8_correction_uses_unquantized_q():
    """The e4m3 path quantizes only the logits: the first-order correction s (q_t Hbar) A_t / D_t
    takes the unquantized q.  Two queries q1 and q1 + delta with the same e4m3 codes and row scales
    (every row's largest entry, which sets its scale, is left alone; the others move by 1%, well
    inside their rounding interval) give identical logits, so the outputs differ only through the
    correction.  With keep_k = 0 and full blocks, A_t / D_t = sum_j alpha / sum_j cnt_j alpha =
    1 / block for every row, so the difference is (s / block) delta Hbar exactly, with Hbar the
    mean over blocks of cnt_j times the biased cross-covariance of the block's k and v (numpy.cov).
    A correction built from the e4m3 copy of q would leave the two outputs equal."""
    r = _rng(43)
    L, d, block, scale = 64, 8, 16, 0.8
    q1 = _representable(r, L, d, 0.003 * (1.0 + r.random(L)))
    delta = 0.01 * q1
    delta[:, 0] = 0.0                       # column 0 holds each row's largest |q| (the code 448)
    k = r.standard_normal((L, d)) * 0.7
    v = r.standard_normal((L, d))
    hbar = np.zeros((d, d))
    for s, e in O.block_bounds(L, block):
        hbar += (e - s) * np.cov(k[s:e].T, v[s:e].T, bias=True)[:d, d:] / (L // block)
    run = lambda qq: O.pisa_fp8(qq[None, None], k[None, None], v[None, None], block, 0, 0.5, scale)["o"][0, 0]
    diff = run(q1 + delta) - run(q1)
    want = (scale / block) * (delta @ hbar)
    err = _rel(diff, want)
    return bool(np.abs(want).max() > 0 and err < 1e-8), f"rel err {err:.3e}"


def pin_dense_attention_is_sdpa():
    """The oracle's textbook dense attention (used as the reference of the dense-attention checks)
    equals torch SDPA in float64, with d != dv, a scale, and logits large enough that an unshifted
    exponential would overflow."""
    worst = 0.0
    for seed, (L, Lk, d, dv), scale, spread in ((50, (37, 53, 6, 4), 0.7, 1.0), (51, (64, 64, 16, 16), 1.0, 9.0)):
        q, k, _ = _qkv(seed, L, d, spread=spread)
        k = _rng(seed + 100).standard_normal((Lk, d)) * spread
        v = _rng(seed + 200).standard_normal((Lk, dv))
        worst = max(worst, _rel(O.dense_attention(q, k, v, scale), _sdpa(q, k, v, scale)))
    return worst < 1e-12, f"max rel err {worst:.3e}"


ALL_PINS = [
    pin_all_selected_is_dense, pin_block_one_is_dense, pin_constant_key_blocks_are_dense,
    pin_exact_only_is_masked_sdpa, pin_brute_force_matches, pin_value_shift_equivariance,
    pin_value_scale_linearity, pin_in_block_permutation, pin_second_order_when_blocks_share_structure,
    pin_first_order_in_general, pin_block_means_and_sums, pin_first_order_matrix_is_cross_covariance,
    pin_global_statistic_closed_form, pin_cov_norm, pin_route_combination_rule, pin_route_count_weighting,
    pin_route_lambda_zero_is_pooled_topk, pin_route_large_lambda_is_cov_topk, pin_route_edges,
    pin_axis_permutation_by_hand, pin_axis_permutation_coordinates,
    pin_permute_rows_inverse_and_dense_equivariance, pin_reordered_pisa_all_selected_is_dense,
    pin_e4m3_by_hand, pin_quantize_groups_bounds, pin_fp8_exact_on_representable_inputs,
    pin_fp8_constant_key_blocks_are_dense, pin_fp8_correction_uses_unquantized_q, pin_dense_attention_is_sdpa,
]
