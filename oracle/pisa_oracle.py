"""Plain fp64 CPU oracle for piecewise sparse attention (PISA).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this module:
only the test suite, the package smoke check and the benchmark's CPU-baseline leg use it.  It shares
no code with the CUDA library (no kernels, headers, helpers or tables) and imports nothing from it.

Source: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers"
(gist.science technical summary of arXiv 2602.01077), cited below as [PISA §n] for its sections
§1 문제 정의 (problem), §2 방법론 (method: 핵심 알고리즘 = core algorithm, the numerator equation,
공분산 인식 라우팅 = covariance-aware routing, 하드웨어 구현 = hardware implementation).

Everything is evaluated per (batch, head) in float64 on inputs already rounded to the run's dtype,
so input rounding is not counted as error.  Notation follows the page: t = query token, i = query
block, j = key block, n = token inside a key block, S_i = critical (exact) blocks, U_i = the rest,
alpha_{t,j} = exp(q_t . kbar_j), Hbar = global first-order statistic, M_j = ||H_j - Hbar||.

Readings taken where the page is silent (each is listed in the design notes):
  * D_t is not printed.  It is built from the same terms as N_t; its first-order term is
    sum_n q_t.(k_n - kbar_j) * alpha = 0 because kbar_j is the block mean, so
    D_t = sum_{S_i} sum_n e^{q.k} + sum_{U_i} cnt_j alpha_{t,j}.
  * H_j = sum_n (k_n - kbar_j)^T v_n  (d x dv, a sum), the first-order coefficient of the Taylor
    expansion of sum_n e^{q.k_n} v_n about kbar_j; Hbar = unweighted mean of H_j over all key blocks.
  * ||.||_2 of a matrix is read as the Frobenius norm (spectral available as a diagnostic).
  * Routing score r_ij = P_ij + lambda * M_j / sum_l M_l, with P_ij the cnt-weighted softmax over j
    of the pooled-query / centroid score; top-k with ties to the lower j, lists ascending.
  * Query blocks use the key-block partition; the softmax scale multiplies every logit and the
    first-order correction.
Parity of the two routing readings (norm choice, score combination) is pinned only by their
special cases (lambda = 0, lambda -> inf, keep_k = nb), not by any number on the page.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "num_blocks", "block_bounds", "block_stats", "route_scores", "route_select",
    "attention_head", "pisa", "dense_attention", "brute_force_head",
    "axis_permutation", "permute_rows", "pisa_reordered",
    "E4M3_MAX", "e4m3", "quantize_groups", "fp8_logit_inputs", "pisa_fp8",
]


# --------------------------------------------------------------------------------------------
# Blocks  [PISA §2 핵심 알고리즘: KV tokens are split into blocks, critical S_i vs uncritical U_i]
# --------------------------------------------------------------------------------------------
def num_blocks(L: int, block: int) -> int:
    """nb = ceil(L / block); the last block may hold fewer than ``block`` tokens."""
    return -(-L // block)


def block_bounds(L: int, block: int) -> List[tuple]:
    """[(start, end)] of each contiguous block; cnt_j = end - start."""
    return [(j * block, min((j + 1) * block, L)) for j in range(num_blocks(L, block))]


# --------------------------------------------------------------------------------------------
# Pre-computation  [PISA §2 하드웨어 구현 step 1; zeroth-order bullet; global first-order bullet]
# --------------------------------------------------------------------------------------------
def _centroid(kk: np.ndarray) -> np.ndarray:
    """kbar_j: mean of the keys of block j (zeroth-order expansion point)."""
    return kk.sum(axis=0) / kk.shape[0]


def _value_sum(vv: np.ndarray) -> np.ndarray:
    """sum_n v_{j,n}: the aggregated value vector of block j (numerator, second term)."""
    return vv.sum(axis=0)


def _first_order_matrix(kk: np.ndarray, vv: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """H_j = sum_n (k_n - kbar_j)^T v_n, d x dv: the block's first-order (covariance) matrix."""
    return (kk - kbar[None, :]).T @ vv


def _global_first_order(H: np.ndarray) -> np.ndarray:
    """Hbar = average of the block-wise first-order matrices over all blocks of the head."""
    return H.sum(axis=0) / H.shape[0]


def _cov_norm(Hj: np.ndarray, Hbar: np.ndarray, norm: str) -> float:
    """M_j = ||H_j - Hbar|| (Frobenius by default; spectral as a diagnostic)."""
    diff = Hj - Hbar
    if norm == "fro":
        return float(np.sqrt((diff * diff).sum()))
    if norm == "spectral":
        return float(np.linalg.norm(diff, ord=2))
    raise ValueError(norm)


def block_stats(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int, norm: str = "fro") -> Dict:
    """Per-head statistics: qbar, kbar, vsum, cnt, H, Hbar, M.  Inputs are [L, d] / [L, dv]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = k.shape
    dv = v.shape[1]
    bounds = block_bounds(L, block)
    nb = len(bounds)
    qbar = np.zeros((nb, d))
    kbar = np.zeros((nb, d))
    vsum = np.zeros((nb, dv))
    cnt = np.zeros(nb, dtype=np.int64)
    H = np.zeros((nb, d, dv))
    for j, (s, e) in enumerate(bounds):
        cnt[j] = e - s
        qbar[j] = _centroid(q[s:e])          # pooled query of query block j (same partition)
        kbar[j] = _centroid(k[s:e])
        vsum[j] = _value_sum(v[s:e])
        H[j] = _first_order_matrix(k[s:e], v[s:e], kbar[j])
    Hbar = _global_first_order(H)
    M = np.array([_cov_norm(H[j], Hbar, norm) for j in range(nb)])
    return dict(qbar=qbar, kbar=kbar, vsum=vsum, cnt=cnt, H=H, Hbar=Hbar, M=M)


# --------------------------------------------------------------------------------------------
# Covariance-aware routing  [PISA §2 공분산 인식 라우팅; §3 contribution 3]
# --------------------------------------------------------------------------------------------
def _block_attention_mass(qbar: np.ndarray, kbar: np.ndarray, cnt: np.ndarray, scale: float) -> np.ndarray:
    """P_ij = cnt_j e^{s q̄_i.k̄_j} / sum_l cnt_l e^{s q̄_i.k̄_l}: zeroth-order attention mass per block."""
    s = scale * (qbar @ kbar.T)
    s = s - s.max(axis=1, keepdims=True)
    w = cnt[None, :].astype(np.float64) * np.exp(s)
    return w / w.sum(axis=1, keepdims=True)


def _normalised_cov(M: np.ndarray) -> np.ndarray:
    """M_j / sum_l M_l (all zeros when every M_j is zero)."""
    tot = M.sum()
    return M / tot if tot > 0 else np.zeros_like(M)


def route_scores(stats: Dict, lam: float, scale: float = 1.0) -> np.ndarray:
    """r_ij = P_ij + lambda * M̃_j, shape [nqb, nb]."""
    P = _block_attention_mass(stats["qbar"], stats["kbar"], stats["cnt"], scale)
    return P + lam * _normalised_cov(stats["M"])[None, :]


def route_select(r: np.ndarray, keep_k: int) -> np.ndarray:
    """S_i: the keep_k largest r_ij per row, ties to the lower j, returned ascending [nqb, keep_k]."""
    nqb, nb = r.shape
    j = np.arange(nb)
    sel = np.zeros((nqb, keep_k), dtype=np.int64)
    for i in range(nqb):
        order = np.lexsort((j, -r[i]))      # primary: larger score; secondary: smaller index
        sel[i] = np.sort(order[:keep_k])
    return sel


# --------------------------------------------------------------------------------------------
# Exact-or-approximate attention  [PISA §2: o_t = N_t / D_t and the numerator equation]
# --------------------------------------------------------------------------------------------
def _correction(qi: np.ndarray, stats: Dict, alpha: np.ndarray, U: Sequence[int], scale: float,
                first_order: str) -> np.ndarray:
    """Third numerator term: scale * q_t Hbar * sum_{j in U_i} alpha_{t,j} (global first order).

    ``first_order='per_block'`` uses each unselected block's own H_j instead (the variant the page
    rejects for memory reasons); it is a diagnostic only.
    """
    if len(U) == 0:
        return np.zeros((qi.shape[0], stats["vsum"].shape[1]))
    if first_order == "global":
        return scale * (qi @ stats["Hbar"]) * alpha.sum(axis=1, keepdims=True)
    if first_order == "per_block":
        out = np.zeros((qi.shape[0], stats["vsum"].shape[1]))
        for c, j in enumerate(U):
            out += scale * alpha[:, c:c + 1] * (qi @ stats["H"][j])
        return out
    if first_order == "none":
        return np.zeros((qi.shape[0], stats["vsum"].shape[1]))
    raise ValueError(first_order)


def _denominator(ez: np.ndarray, alpha: np.ndarray, cnt_u: np.ndarray) -> np.ndarray:
    """D_t = sum_{S_i} sum_n e^{q.k} + sum_{U_i} cnt_j alpha_{t,j} (first-order term is zero)."""
    return ez.sum(axis=1) + alpha @ cnt_u.astype(np.float64)


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int, sel: np.ndarray,
                   stats: Dict, scale: float = 1.0, mode: str = "pisa",
                   first_order: str = "global", qblocks: Optional[Sequence[int]] = None,
                   q_corr: Optional[np.ndarray] = None) -> np.ndarray:
    """o = N / D for one head; ``mode='exact_only'`` drops U_i (the keep-or-drop baseline).

    ``qblocks`` restricts the evaluation to those query blocks (other rows are NaN).  ``q_corr``,
    when given, is the query used by the first-order correction (the logits use ``q``).
    """
    qc_all = None if q_corr is None else np.asarray(q_corr, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L = q.shape[0]
    bounds = block_bounds(L, block)
    nb = len(bounds)
    o = np.zeros((L, v.shape[1])) if qblocks is None else np.full((L, v.shape[1]), np.nan)
    wanted = range(nb) if qblocks is None else sorted(set(int(i) for i in qblocks))
    for i in wanted:
        qs, qe = bounds[i]
        S = [int(j) for j in sel[i]]
        Sset = set(S)
        U = [j for j in range(nb) if j not in Sset] if mode == "pisa" else []
        qi = q[qs:qe]
        tok = np.concatenate([np.arange(*bounds[j]) for j in S]) if S else np.zeros(0, dtype=np.int64)
        z = scale * (qi @ k[tok].T)                                  # exact logits
        c = scale * (qi @ stats["kbar"][U].T) if U else np.zeros((qi.shape[0], 0))
        m = np.full(qi.shape[0], -np.inf)
        if z.shape[1]:
            m = np.maximum(m, z.max(axis=1))
        if c.shape[1]:
            m = np.maximum(m, c.max(axis=1))                         # shift: inert, avoids overflow
        ez = np.exp(z - m[:, None])
        alpha = np.exp(c - m[:, None])
        N = ez @ v[tok]                                               # exact sparse term
        if U:
            N = N + alpha @ stats["vsum"][U]                          # block-wise zeroth order
            qc = qi if qc_all is None else qc_all[qs:qe]
            N = N + _correction(qc, stats, alpha, U, scale, first_order)
        D = _denominator(ez, alpha, stats["cnt"][U] if U else np.zeros(0))
        o[qs:qe] = N / D[:, None]
    return o


def pisa(q, k, v, block: int, keep_k: int, lam: float, scale: float = 1.0, mode: str = "pisa",
         first_order: str = "global", norm: str = "fro", heads: Optional[Sequence[int]] = None,
         qblocks: Optional[Sequence[int]] = None) -> Dict:
    """Whole pipeline on [B, H, L, d] inputs: stats -> route -> attention, per (batch, head).

    Returns dict with o [B,H,L,dv], sel [B,H,nqb,keep_k], scores r [B,H,nqb,nb] and the stats
    arrays stacked over (B, H).  ``heads`` selects which head indices of the input to evaluate;
    ``qblocks`` restricts the attention output to those query blocks (statistics and routing are
    always complete).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hh, L, d = q.shape
    hs = list(range(Hh)) if heads is None else list(heads)
    out: Dict[str, list] = {key: [] for key in ("o", "sel", "r", "qbar", "kbar", "vsum", "Hbar", "M", "cnt")}
    for b in range(B):
        row = {key: [] for key in out}
        for h in hs:
            st = block_stats(q[b, h], k[b, h], v[b, h], block, norm)
            r = route_scores(st, lam, scale)
            sel = route_select(r, keep_k)
            o = attention_head(q[b, h], k[b, h], v[b, h], block, sel, st, scale, mode, first_order, qblocks)
            for key, val in (("o", o), ("sel", sel), ("r", r), ("qbar", st["qbar"]), ("kbar", st["kbar"]),
                             ("vsum", st["vsum"]), ("Hbar", st["Hbar"]), ("M", st["M"]), ("cnt", st["cnt"])):
                row[key].append(val)
        for key in out:
            out[key].append(np.stack(row[key]))
    return {key: np.stack(val) for key, val in out.items()}


# --------------------------------------------------------------------------------------------
# Independent evaluators used to pin the above
# --------------------------------------------------------------------------------------------
def dense_attention(q, k, v, scale: float = 1.0) -> np.ndarray:
    """Textbook softmax(scale Q K^T) V for one head, fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * (q @ k.T)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def brute_force_head(q, k, v, block: int, sel, scale: float = 1.0, first_order: str = "global") -> np.ndarray:
    """Literal per-token evaluation (pure Python loops; meant for L <= 256).

    Unselected blocks contribute the first-order Taylor expansion of e^{s q_t.k_n} about kbar_j,
    token by token: e^{s q.kbar} (1 + s q.(k_n - kbar)) v_n in the numerator and the same weight in
    the denominator (whose first-order part must cancel).  With ``first_order='global'`` the
    block's first-order numerator term is replaced by the hybrid-order global one built from Hbar,
    which is itself accumulated here by explicit loops.  No max shift is applied.
    """
    q = [list(map(float, row)) for row in np.asarray(q, dtype=np.float64)]
    k = [list(map(float, row)) for row in np.asarray(k, dtype=np.float64)]
    v = [list(map(float, row)) for row in np.asarray(v, dtype=np.float64)]
    L, d, dv = len(q), len(q[0]), len(v[0])
    nb = -(-L // block)
    members = [list(range(j * block, min((j + 1) * block, L))) for j in range(nb)]
    kbar = []
    for j in range(nb):
        kbar.append([sum(k[n][a] for n in members[j]) / len(members[j]) for a in range(d)])
    Hbar = [[0.0] * dv for _ in range(d)]
    for j in range(nb):
        for n in members[j]:
            for a in range(d):
                dk = k[n][a] - kbar[j][a]
                for c in range(dv):
                    Hbar[a][c] += dk * v[n][c] / nb

    def dot(x, y):
        return sum(xa * ya for xa, ya in zip(x, y))

    out = np.zeros((L, dv))
    for t in range(L):
        i = t // block
        chosen = set(int(x) for x in sel[i])
        Nt = [0.0] * dv
        Dt = 0.0
        for j in range(nb):
            if j in chosen:
                for n in members[j]:
                    w = math.exp(scale * dot(q[t], k[n]))
                    Dt += w
                    for c in range(dv):
                        Nt[c] += w * v[n][c]
            else:
                a0 = math.exp(scale * dot(q[t], kbar[j]))
                for n in members[j]:
                    lin = scale * sum(q[t][a] * (k[n][a] - kbar[j][a]) for a in range(d))
                    Dt += a0 * (1.0 + lin)
                    for c in range(dv):
                        Nt[c] += a0 * v[n][c]
                        if first_order == "per_block":
                            Nt[c] += a0 * lin * v[n][c]
                if first_order == "global":
                    for c in range(dv):
                        Nt[c] += a0 * scale * sum(q[t][a] * Hbar[a][c] for a in range(d))
        out[t] = [x / Dt for x in Nt]
    return out


# --------------------------------------------------------------------------------------------
# Token reordering before blocking
# ["PAROAttention: Pattern-Aware ReOrdering for Efficient Sparse and Quantized Attention in Visual
#  Generation Models", abstract: tokens are reordered so that attention becomes block-wise.  The
#  page gives no algorithm; the reading here permutes the axis order of the frames x height x width
#  token grid, and the same permutation is applied to q, k and v and undone on the output.]
# --------------------------------------------------------------------------------------------
def axis_permutation(grid, order: str, extra_tokens: int = 0) -> np.ndarray:
    """perm[i] = raster index (t slowest, then h, then w) of the token at position i when the grid
    is listed with the axes in ``order`` (slowest first); extra tokens keep their place at the end."""
    T, Hg, W = grid
    if sorted(order) != ["h", "t", "w"]:
        raise ValueError(order)
    raster = np.arange(T * Hg * W).reshape(T, Hg, W)
    axes = tuple("thw".index(c) for c in order)
    grid_part = np.transpose(raster, axes).reshape(-1)
    return np.concatenate([grid_part, np.arange(T * Hg * W, T * Hg * W + extra_tokens)]).astype(np.int64)


def permute_rows(x: np.ndarray, perm: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Gather rows along axis -2 (out[..., i, :] = x[..., perm[i], :]) or, with inverse, scatter
    them back (out[..., perm[i], :] = x[..., i, :])."""
    x = np.asarray(x)
    if not inverse:
        return x[..., perm, :]
    out = np.empty_like(x)
    out[..., perm, :] = x
    return out


def pisa_reordered(q, k, v, perm, block: int, keep_k: int, lam: float, scale: float = 1.0, **kw) -> Dict:
    """PISA on the reordered sequence, output put back in the original token order."""
    r = pisa(permute_rows(q, perm), permute_rows(k, perm), permute_rows(v, perm), block, keep_k, lam, scale, **kw)
    r["o"] = permute_rows(r["o"], perm, inverse=True)
    return r


# --------------------------------------------------------------------------------------------
# e4m3 logits for the exact stage (low-bit attention in the spirit of the INT8/INT4 attention that
# "PAROAttention: Pattern-Aware ReOrdering ..." mentions in its abstract; no page gives an FP8
# recipe, so this is a reading).  The
# exact and zeroth-order logits use e4m3 copies of q (one scale per row), k (one scale per key
# block) and kbar (one scale per tile of 128 centroids); the scale of a group is max|x| / 448 and
# the code of x is e4m3(x / scale), both decided in float32.  Routing, the values and the
# first-order correction keep the unquantized inputs.
# --------------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3(x: np.ndarray) -> np.ndarray:
    """Round float32 values (|x| <= 448) to the nearest e4m3 value, ties to even (torch's
    float8_e4m3fn conversion on the CPU, a library primitive); returned as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def quantize_groups(x: np.ndarray, group_of_row: np.ndarray):
    """Per-group scale s_g = float32(max|x| over the group's rows) / 448 (1 for an all-zero group)
    and dequantized values e4m3(x / s_g) * s_g.  Returns (dequantized float64, scales float32)."""
    x32 = np.asarray(x, dtype=np.float32)
    ngroups = int(group_of_row.max()) + 1 if len(group_of_row) else 0
    amax = np.zeros(ngroups, dtype=np.float32)
    np.maximum.at(amax, group_of_row, np.abs(x32).max(axis=1))
    sc = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    codes = e4m3((x32 / sc[group_of_row][:, None]).astype(np.float32))
    return codes * sc[group_of_row][:, None].astype(np.float64), sc


def fp8_logit_inputs(q: np.ndarray, k: np.ndarray, kbar: np.ndarray, block: int):
    """Dequantized e4m3 copies of q (per row), k (per key block) and kbar (per 128 centroids)."""
    L = q.shape[0]
    nb = kbar.shape[0]
    qd, _ = quantize_groups(q, np.arange(L))
    kd, _ = quantize_groups(k, np.arange(L) // block)
    kbd, _ = quantize_groups(kbar, np.arange(nb) // 128)
    return qd, kd, kbd


def pisa_fp8(q, k, v, block: int, keep_k: int, lam: float, scale: float = 1.0, mode: str = "pisa",
             heads: Optional[Sequence[int]] = None, qblocks: Optional[Sequence[int]] = None) -> Dict:
    """pisa() with the attention logits computed from the e4m3 copies (see above)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hh, L, d = q.shape
    hs = list(range(Hh)) if heads is None else list(heads)
    out: Dict[str, list] = {key: [] for key in ("o", "sel", "r")}
    for b in range(B):
        row = {key: [] for key in out}
        for h in hs:
            st = block_stats(q[b, h], k[b, h], v[b, h], block)
            r = route_scores(st, lam, scale)
            sel = route_select(r, keep_k)
            qd, kd, kbd = fp8_logit_inputs(q[b, h], k[b, h], st["kbar"], block)
            st_l = dict(st)
            st_l["kbar"] = kbd
            o = attention_head(qd, kd, v[b, h], block, sel, st_l, scale, mode, "global", qblocks, q_corr=q[b, h])
            for key, val in (("o", o), ("sel", sel), ("r", r)):
                row[key].append(val)
        for key in out:
            out[key].append(np.stack(row[key]))
    return {key: np.stack(val) for key, val in out.items()}
