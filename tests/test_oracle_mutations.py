"""Plant plausible mistakes in the oracle (on the CPU) and check that some pin catches each one.

A mistake that no pin notices would mean the pins do not constrain that part of the oracle.
"""
import numpy as np
import pytest

from oracle import pisa_oracle as O
from tests import oracle_pins as P


def _corr_sign(qi, stats, alpha, U, scale, first_order):
    return -_ORIG["_correction"](qi, stats, alpha, U, scale, first_order)


def _corr_zero(qi, stats, alpha, U, scale, first_order):
    return 0.0 * _ORIG["_correction"](qi, stats, alpha, U, scale, first_order)


def _corr_transposed(qi, stats, alpha, U, scale, first_order):
    st = dict(stats)
    st["Hbar"] = stats["Hbar"].T
    st["H"] = np.swapaxes(stats["H"], 1, 2)
    return _ORIG["_correction"](qi, st, alpha, U, scale, first_order)


def _corr_unscaled(qi, stats, alpha, U, scale, first_order):
    return _ORIG["_correction"](qi, stats, alpha, U, 1.0, first_order)


MUTATIONS = {
    "correction dropped": ("_correction", _corr_zero),
    "correction sign flipped": ("_correction", _corr_sign),
    "correction uses H transposed": ("_correction", _corr_transposed),
    "correction misses softmax scale": ("_correction", _corr_unscaled),
    "denominator misses cnt_j": ("_denominator", lambda ez, a, c: ez.sum(axis=1) + a.sum(axis=1)),
    "H_j not centred": ("_first_order_matrix", lambda kk, vv, kbar: kk.T @ vv),
    "Hbar is a sum": ("_global_first_order", lambda H: H.sum(axis=0)),
    "centroid is first token": ("_centroid", lambda kk: kk[0].copy()),
    "value sum is a mean": ("_value_sum", lambda vv: vv.mean(axis=0)),
    "route mass ignores cnt": ("_block_attention_mass",
                               lambda qb, kb, cnt, s: _ORIG["_block_attention_mass"](qb, kb, np.ones_like(cnt), s)),
    "M not normalised": ("_normalised_cov", lambda M: M),
    "M squared": ("_cov_norm", lambda Hj, Hb, norm: _ORIG["_cov_norm"](Hj, Hb, norm) ** 2),
}
_ORIG = {name: getattr(O, name) for name, _ in MUTATIONS.values()}


def _tie_high(r, keep_k):
    nqb, nb = r.shape
    out = np.zeros((nqb, keep_k), dtype=np.int64)
    for i in range(nqb):
        order = np.lexsort((-np.arange(nb), -r[i]))
        out[i] = np.sort(order[:keep_k])
    return out


MUTATIONS["ties to the higher index"] = ("route_select", _tie_high)
_ORIG["route_select"] = O.route_select


def _axes_reversed(grid, order, extra_tokens=0):
    return _ORIG["axis_permutation"](grid, order[::-1], extra_tokens)


def _gather_is_scatter(x, perm, inverse=False):
    return _ORIG["permute_rows"](x, perm, not inverse)


MUTATIONS["axis order read fastest first"] = ("axis_permutation", _axes_reversed)
MUTATIONS["gather and scatter swapped"] = ("permute_rows", _gather_is_scatter)
_ORIG["axis_permutation"] = O.axis_permutation
_ORIG["permute_rows"] = O.permute_rows


def _k_per_row(q, k, kbar, block):
    qd, _, kbd = _ORIG["fp8_logit_inputs"](q, k, kbar, block)
    kd, _ = O.quantize_groups(k, np.arange(k.shape[0]))
    return qd, kd, kbd


def _q_per_block(q, k, kbar, block):
    _, kd, kbd = _ORIG["fp8_logit_inputs"](q, k, kbar, block)
    qd, _ = O.quantize_groups(q, np.arange(q.shape[0]) // block)
    return qd, kd, kbd


MUTATIONS["e4m3 k scaled per row"] = ("fp8_logit_inputs", _k_per_row)
MUTATIONS["e4m3 q scaled per block"] = ("fp8_logit_inputs", _q_per_block)


def _bf16_not_e4m3(x):
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


MUTATIONS["e4m3 rounding is bf16 rounding"] = ("e4m3", _bf16_not_e4m3)
_ORIG["fp8_logit_inputs"] = O.fp8_logit_inputs
_ORIG["e4m3"] = O.e4m3



def _corr_from_logit_q(*args, q_corr=None, **kw):
    # the e4m3 path's correction built from the quantized q that the logits use
    return _ORIG["attention_head"](*args, **kw)


def _dense_wrong_axis(q, k, v, scale=1.0):
    s = scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)
    p = np.exp(s - s.max(axis=0, keepdims=True))
    return (p / p.sum(axis=0, keepdims=True)) @ np.asarray(v, np.float64)


MUTATIONS["e4m3 correction uses the quantized q"] = ("attention_head", _corr_from_logit_q)
MUTATIONS["dense attention normalised over queries"] = ("dense_attention", _dense_wrong_axis)
_ORIG["attention_head"] = O.attention_head
_ORIG["dense_attention"] = O.dense_attention

def _caught():
    failed = []
    for pin in P.ALL_PINS:
        try:
            ok, _ = pin()
        except Exception:          # a crash under the planted mistake counts as a catch
            ok = False
        if not ok:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = _caught()
    assert failed, f"no pin caught the planted mistake: {name}"
