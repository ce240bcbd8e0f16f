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
