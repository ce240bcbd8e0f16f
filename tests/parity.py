"""Comparison helpers for CUDA-vs-oracle parity tests.

Tolerances (fixed by the method's accuracy contract, not tuned):
  * selected-block sets must match exactly, except where the oracle's route scores of the
    differing blocks lie within 1e-4 (relative) of the keep_k-th largest score (a near-tie);
  * bf16 inputs: output relative L2 error <= 1e-2 and max-abs error <= 2e-2 * RMS(o), the latter
    counted beyond each element's own rounding to the bf16 output (unit roundoff 2^-8 * |o|):
    rounding the exact fp64 result to bf16 alone reaches 5.5e-2 * RMS on the image workload, whose
    few large rows sit ~20x above the RMS, so the bound can only apply to the arithmetic error;
  * fp32 inputs: output relative L2 error <= 1e-4.
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-4
BF16_REL_L2 = 1e-2
BF16_MAX_ABS_OVER_RMS = 2e-2
BF16_UNIT_ROUNDOFF = 2.0 ** -8
FP32_REL_L2 = 1e-4


def compare_selection(gpu_sel: np.ndarray, ref_sel: np.ndarray, ref_r: np.ndarray, keep_k: int):
    """Returns (bad_rows, tie_rows) for [nqb, keep_k] selections of one head."""
    bad, ties = [], []
    if keep_k == 0:
        return bad, ties
    for i in range(ref_sel.shape[0]):
        g = set(int(x) for x in gpu_sel[i])
        r = set(int(x) for x in ref_sel[i])
        if g == r:
            continue
        if len(g) != keep_k:
            bad.append(i)
            continue
        kth = np.sort(ref_r[i])[::-1][keep_k - 1]
        diff = g ^ r
        if all(abs(ref_r[i][j] - kth) <= TIE_REL * abs(kth) for j in diff):
            ties.append(i)
        else:
            bad.append(i)
    return bad, ties


def output_errors(o_gpu: np.ndarray, o_ref: np.ndarray, rows_mask=None, output_roundoff: float = 0.0):
    """(relative L2, max-abs / RMS(o_ref)) over the rows where rows_mask is True (default all).

    ``output_roundoff`` discounts from each element's error the rounding of the output itself.
    """
    a = np.asarray(o_gpu, dtype=np.float64)
    b = np.asarray(o_ref, dtype=np.float64)
    if rows_mask is not None:
        a = a[rows_mask]
        b = b[rows_mask]
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    rms = float(np.sqrt(np.mean(b * b)))
    excess = np.maximum(np.abs(a - b) - output_roundoff * np.abs(b), 0.0)
    mx = float(excess.max() / max(rms, 1e-300)) if a.size else 0.0
    return rel, mx


def assert_output(o_gpu, o_ref, dtype: str, rows_mask=None, what=""):
    rel, mx = output_errors(o_gpu, o_ref, rows_mask, BF16_UNIT_ROUNDOFF if dtype == "bf16" else 0.0)
    if dtype == "fp32":
        assert rel <= FP32_REL_L2, f"{what}: fp32 rel-L2 {rel:.3e} > {FP32_REL_L2}"
    else:
        assert rel <= BF16_REL_L2, f"{what}: bf16 rel-L2 {rel:.3e} > {BF16_REL_L2}"
        assert mx <= BF16_MAX_ABS_OVER_RMS, f"{what}: bf16 max-abs/RMS {mx:.3e} > {BF16_MAX_ABS_OVER_RMS}"
    return rel, mx


def rows_of_blocks(L: int, block: int, blocks) -> np.ndarray:
    m = np.zeros(L, dtype=bool)
    for i in blocks:
        m[i * block:min((i + 1) * block, L)] = True
    return m
