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
