"""bench.py's multi-rank path on CPU: two gloo ranks, 127.0.0.1 rendezvous."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv
        mx, sm = bench.aggregate([1.0 + rank, 10.0 - rank], [2.0 * (rank + 1)], torch.device("cpu"), world)
        w = WORKLOADS["tiny-fp32"].with_(heads=1)
        qt, _, _ = make_qkv(w, seed=bench.rank_seed(w, rank))
        firsts = [torch.zeros(4) for _ in range(world)]
        dist.all_gather(firsts, qt.flatten()[:4].contiguous())
        distinct = not torch.equal(firsts[0], firsts[1])
        out_q.put((rank, mx, sm, distinct))
    finally:
        dist.destroy_process_group()


def test_two_ranks_aggregate_max_time_and_sum_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, distinct in out:
        assert mx == [2.0, 10.0]          # slowest rank's time
        assert sm == [6.0]                # work summed over ranks (2 + 4)
        assert distinct                   # ranks draw different batch elements


def test_single_rank_aggregate_is_identity():
    import bench
    assert bench.aggregate([3.0], [5.0], torch.device("cpu"), 1) == ([3.0], [5.0])


def test_reference_arm_runs_on_rank0_only():
    import argparse

    import bench
    args = argparse.Namespace(workload="tiny-fp32", steps=1, warmup=0)
    assert bench.run_reference(args, rank=1, world=2) is None
    res = bench.run_reference(args, rank=0, world=2)
    assert res["impl"] == "reference" and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["value"] > 0


def _seq_shard_worker(rank, world, port, out_q):
    """One head's key and query blocks split across ranks: each rank reduces the statistics of its
    own blocks, then one all-reduce (the d x dv partial sums of H_j) and one all-gather (k̄, vsum,
    cnt, M, q̄) give every rank the head's full statistics for routing and attention."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import numpy as np
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import pisa_oracle as O
        from piecewise_approximate_attention_b200.workloads import WORKLOADS, make_qkv
        w = WORKLOADS["tiny-fp32"].with_(heads=1, grid=(15, 8, 9))      # L 1080: 17 blocks, the last of 56
        q, k, v = (x[0, 0].double().numpy() for x in make_qkv(w))
        L, block, nb = w.seq_len, w.block, w.num_blocks
        per = -(-nb // world)
        j0, j1 = rank * per, min(nb, (rank + 1) * per)
        sl = slice(j0 * block, min(j1 * block, L))
        loc = O.block_stats(q[sl], k[sl], v[sl], block)
        # exchange: sum of H_j over all blocks, then the per-block vectors of every rank
        hsum = torch.from_numpy(loc["H"].sum(axis=0))
        dist.all_reduce(hsum)
        hbar = hsum.numpy() / nb
        m_loc = np.array([np.linalg.norm(loc["H"][j] - hbar) for j in range(j1 - j0)])

        def gather(a):
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
            pad = torch.zeros((per,) + tuple(t.shape[1:]), dtype=torch.float64)
            pad[: t.shape[0]] = t
            parts = [torch.zeros_like(pad) for _ in range(world)]
            dist.all_gather(parts, pad)
            return torch.cat(parts)[:nb].numpy()

        st = dict(qbar=gather(loc["qbar"]), kbar=gather(loc["kbar"]), vsum=gather(loc["vsum"]),
                  cnt=gather(loc["cnt"]).astype(np.int64), M=gather(m_loc), Hbar=hbar)
        r = O.route_scores(st, w.lam)
        sel = O.route_select(r, w.keep_k)
        mine = list(range(j0, j1))
        o = O.attention_head(q, k, v, block, sel, st, qblocks=mine)
        ref = O.pisa(q[None, None], k[None, None], v[None, None], block, w.keep_k, w.lam)
        rows = slice(j0 * block, min(j1 * block, L))
        ok_sel = np.array_equal(sel[j0:j1], ref["sel"][0, 0][j0:j1])
        err_o = float(np.abs(o[rows] - ref["o"][0, 0][rows]).max())
        err_m = float(np.abs(st["M"] - ref["M"][0, 0]).max() / np.abs(ref["M"][0, 0]).max())
        out_q.put((rank, ok_sel, err_o, err_m))
    finally:
        dist.destroy_process_group()


def test_sequence_sharded_statistics_match_one_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_sel, err_o, err_m in out:
        assert ok_sel, rank
        assert err_m < 1e-12, (rank, err_m)
        assert err_o < 1e-12, (rank, err_o)
