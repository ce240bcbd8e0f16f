"""Writes tests/golden/tiny_fp32.json from the fp64 oracle alone (no GPU code is imported).

Run from the repository root:  python tests/golden/make_golden.py
The fixture freezes the oracle's output on the 2-head, L=1024, d=64, block-64 workload so that an
unintended change to the oracle's arithmetic or to the input generator shows up as a test failure.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import pisa_oracle as O                                    # noqa: E402
from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv  # noqa: E402


def summarise():
    w = WORKLOADS["tiny-fp32"]
    q, k, v = (t.double().numpy() for t in make_qkv(w))
    res = O.pisa(q, k, v, w.block, w.keep_k, w.lam)
    o = res["o"]
    return {
        "workload": w.name, "block": w.block, "keep_k": w.keep_k, "lam": w.lam,
        "sel": res["sel"].tolist(),
        "M": np.round(res["M"], 12).tolist(),
        "o_sum": float(o.sum()), "o_sumsq": float((o * o).sum()),
        "o_samples": [[int(h), int(t), int(c), float(o[0, h, t, c])]
                      for h, t, c in [(0, 0, 0), (0, 511, 17), (1, 1023, 63), (1, 300, 5)]],
        "Hbar_trace": [float(np.trace(res["Hbar"][0, h])) for h in range(w.heads)],
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32.json")
    with open(path, "w") as f:
        json.dump(summarise(), f, indent=1)
    print("wrote", path)
