"""Synthetic input generator: determinism, shapes, head-subset consistency, config sizes."""
import numpy as np
import torch

from piecewise_approximate_attention_b200.workloads import WORKLOADS, Workload, _field, make_qkv


def test_config_sizes():
    w = WORKLOADS
    assert (w["tiny-fp32"].seq_len, w["tiny-fp32"].num_blocks, w["tiny-fp32"].keep_k) == (1024, 16, 4)
    assert (w["image-dit"].seq_len, w["image-dit"].num_blocks, w["image-dit"].keep_k) == (4608, 72, 18)
    assert (w["video-dit-small"].seq_len, w["video-dit-small"].num_blocks, w["video-dit-small"].keep_k) == (32760, 512, 64)
    assert (w["video-dit-large"].seq_len, w["video-dit-large"].num_blocks, w["video-dit-large"].keep_k) == (75600, 591, 74)
    assert w["sweep-L131072-s0.9375"].keep_k == 128 and w["sweep-L8192-s0"].keep_k == 128


def test_deterministic_and_subset_consistent():
    w = Workload("t", 1, 3, (2, 8, 8), 16, 64, 64, 0.5, 0.5, "bf16", seed=5)
    a = make_qkv(w)
    b = make_qkv(w, heads=[2])
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 3, 144, 64)
        assert torch.equal(x[:, 2:3], y)
    c = make_qkv(w, seed=6)
    assert not torch.equal(a[0], c[0])


def test_field_unit_rms_and_scale_folded():
    F = _field(np.random.default_rng(0), (8, 32, 32), 128)
    assert 0.7 < np.sqrt((F ** 2).mean()) < 1.4
    w = Workload("t", 1, 1, (4, 16, 16), 0, 128, 64, 0.5, 0.5, "fp32")
    q, k, v = make_qkv(w)
    # q carries the 1/sqrt(d) scale; k and v do not
    assert 0.05 < q.std().item() < 0.15 and 0.8 < k.std().item() < 1.5 and 0.9 < v.std().item() < 1.1
