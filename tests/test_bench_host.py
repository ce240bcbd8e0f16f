"""Host-side pieces of bench.py (no GPU): the kernel-code digest that ties a committed ncu summary
to the kernel source it was taken on."""
import os

import bench


def test_code_digest_ignores_comments_and_whitespace(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("// header\n__global__ void k(int* x) {\n  x[0] = 1;   // one\n}\n")
    b.write_text("/* another header */\n__global__   void k(int* x) {\n\n  x[0] = 1;\n}\n")
    c.write_text("__global__ void k(int* x) {\n  x[0] = 2;\n}\n")
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))


def test_profiled_traffic_is_an_integer_or_none():
    t = bench._profiled_traffic("video-dit-large")
    assert t is None or (isinstance(t, int) and t > 0)
    assert bench._profiled_traffic("no-such-workload") is None


def test_effective_flops_counts_selected_blocks_by_hand():
    """4 d sum_i n_i sum_{j in S_i} cnt_j for the exact part, 4 d L (nb - keep_k) for the centroid
    part, on a 150-token head with 64-token blocks (cnt = 64, 64, 22)."""
    import torch
    sel = torch.tensor([[[[0, 1], [1, 2], [0, 2]]]], dtype=torch.int32)
    exact, centroid = bench.effective_flops(sel, 150, 64, 8, 3)
    assert exact == 4 * 8 * (64 * (64 + 64) + 64 * (64 + 22) + 22 * (64 + 22))
    assert centroid == 4 * 8 * 150 * (3 - 2)
