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


def test_summaries_of_interleaved_arms():
    """Median / p10 / p90 of an arm's times and the per-rep ratio of two interleaved arms."""
    a = [(float(x), 1800.0) for x in (10, 11, 12, 13, 14, 15, 16, 17, 18, 19)]
    b = [(float(x), 1700.0) for x in (8, 10, 12, 12, 14, 10, 16, 17, 9, 19)]
    s = bench.summarize(a)
    assert s["median_ms"] == 14.5 and s["n"] == 10 and s["sm_mhz"] == 1800.0
    assert s["p10_ms"] == 10.9 and s["p90_ms"] == 18.1
    r = bench.ratio_summary(a, b)
    per_rep = sorted(x[0] / y[0] - 1.0 for x, y in zip(a, b))
    assert r["n"] == 10 and abs(r["median"] - round((per_rep[4] + per_rep[5]) / 2, 4)) < 1e-12
    assert bench.summarize([(2.0, None)])["sm_mhz"] is None


def test_time_arms_interleaves_and_skips(monkeypatch):
    """time_arms runs the arms round-robin (A B C A B C ...), each n-th rep for `every`, after the
    warm-up calls; the timing itself goes through CUDA events, faked here."""
    import types
    calls = []

    class Ev:
        def __init__(self, enable_timing=False):
            self.t = 0.0

        def record(self, stream=None):
            self.t = float(len(calls))

        def synchronize(self):
            pass

        def elapsed_time(self, other):
            return other.t - self.t

    fake = types.SimpleNamespace(cuda=types.SimpleNamespace(Event=Ev, synchronize=lambda: None))
    monkeypatch.setitem(__import__("sys").modules, "torch", fake)
    arms = {"a": lambda: calls.append("a"), "b": lambda: calls.append("b"), "d": lambda: calls.append("d")}
    out = bench.time_arms(arms, 4, None, clock=None, every={"d": 2}, warmup=1)
    assert calls[:3] == ["a", "b", "d"]                           # warm-up, once each
    assert calls[3:] == ["a", "b", "d", "a", "b", "a", "b", "d", "a", "b"]
    assert [len(out[k]) for k in "abd"] == [4, 4, 2]
    assert all(ms == 1.0 and mhz is None for ms, mhz in out["a"])
