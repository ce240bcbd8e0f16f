"""Runs the PISA hot path a few times on one workload, for profilers (ncu) to capture.

    python -m piecewise_approximate_attention_b200.profile_case --workload video-dit-large --heads 8 --iters 3
"""
from __future__ import annotations

import argparse


def main():
    import torch

    from .runtime import Pisa
    from .workloads import WORKLOADS, make_qkv

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="video-dit-large")
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    w = WORKLOADS[a.workload].with_(heads=a.heads)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, w.dtype, 1.0, "cuda")
    o = torch.empty_like(q)
    for _ in range(a.iters):
        p(q, k, v, o)
    torch.cuda.synchronize()
    st = p.device_error()
    print(f"{w.name} heads={H} L={L} block={w.block} keep_k={w.keep_k} iters={a.iters} status={st}")
    if st[0] != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
