"""Runs the PISA hot path a few times on one workload, for profilers (ncu) to capture.

    python -m piecewise_approximate_attention_b200.profile_case --workload video-dit-large --heads 8 --iters 3
    python -m piecewise_approximate_attention_b200.profile_case --heads 4 --iters 2 --mode per_block
    python -m piecewise_approximate_attention_b200.profile_case --heads 8 --iters 2 --dtype bf16_fp8qk --reorder hwt
"""
from __future__ import annotations

import argparse


def main():
    import torch

    from . import _lib as C
    from .runtime import Pisa, reorder_tokens, restore_tokens
    from .workloads import WORKLOADS, make_qkv

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="video-dit-large")
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--mode", choices=("pisa", "per_block"), default="pisa")
    ap.add_argument("--dtype", choices=("bf16", "bf16_fp8qk"), default="bf16")
    ap.add_argument("--reorder", default=None, help="axis order of the frames x height x width grid, e.g. hwt")
    a = ap.parse_args()
    mode = C.PISA_MODE_PER_BLOCK if a.mode == "per_block" else C.PISA_MODE_PISA
    w = WORKLOADS[a.workload].with_(heads=a.heads)
    q, k, v = (x.cuda() for x in make_qkv(w))
    B, H, L, d = q.shape
    p = Pisa(B, H, L, d, w.block, w.keep_k, w.lam, a.dtype, 1.0, "cuda", mode)
    o = torch.empty_like(q)
    perm = None
    if a.reorder:
        perm = torch.from_numpy(C.pisa_axis_permutation(w.grid, a.reorder, w.text_tokens)).cuda()
        bufs = [torch.empty_like(q) for _ in range(3)]
        o_r = torch.empty_like(q)
    for _ in range(a.iters):
        if perm is None:
            p(q, k, v, o)
        else:
            for x, b in zip((q, k, v), bufs):
                reorder_tokens(x, perm, out=b)
            p(*bufs, o_r)
            restore_tokens(o_r, perm, out=o)
    torch.cuda.synchronize()
    st = p.device_error()
    print(f"{w.name} heads={H} L={L} block={w.block} keep_k={w.keep_k} mode={a.mode} dtype={a.dtype} reorder={a.reorder} iters={a.iters} status={st}")
    if st[0] != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
