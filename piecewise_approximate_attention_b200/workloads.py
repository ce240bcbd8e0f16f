"""Seeded synthetic inputs shaped like the attention layers of diffusion transformers.

This module only draws numbers: it holds none of the attention method's arithmetic, so both the
CUDA path and the CPU oracle can be fed from it.  Inputs stand in for the DiT workloads (Wan2.1,
HunyuanVideo, FLUX.1, SD 3.5) that "PISA: Piecewise Sparse Attention Is Wiser for Efficient
Diffusion Transformers" evaluates on (§4 실험 결과); none of those models or their activations are used.

Recipe, per (batch, head), from its own counter-seeded PCG64 stream ``default_rng([seed, b, h])``:

1. omega ~ U[0.5, 4.0]^(4x3)   cycles per grid extent, per axis (t, y, x)
   phi   ~ U[0, 2*pi)^(4xd)    phase per sinusoid and channel
   a     ~ N(0, 1)^(4xd)       amplitude per sinusoid and channel
2. F_c(t,y,x) = 2^-1/2 * sum_m a[m,c] * sin(2*pi*(omega[m,0]*t/T + omega[m,1]*y/Hg + omega[m,2]*x/W) + phi[m,c])
   (unit RMS per channel in expectation; tokens in raster order t, y, x)
3. eps_q, eps_k, v ~ N(0, 1)^(Lxd)
4. q = (0.5*F + eps_q) / sqrt(d)   (softmax scale folded into q)
   k =  0.5*F + eps_k               (the same field F as q)
5. cast to the run's dtype (round to nearest even).

Text tokens (image workload only) follow the image tokens with i.i.d. N(0,1) q, k, v (q / sqrt(d)).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "keep_from_sparsity", "make_head", "make_qkv", "to_dtype",
           "make_block_structured"]


def keep_from_sparsity(nb: int, sparsity: float) -> int:
    """Blocks kept per query block for a sparsity fraction: ceil((1 - sparsity) * nb)."""
    return int(math.ceil((1.0 - sparsity) * nb - 1e-9))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    grid: Tuple[int, int, int]          # (T, Hg, W) of the smooth-field tokens
    text_tokens: int
    head_dim: int
    block: int
    sparsity: float                     # fraction of key blocks NOT computed exactly
    lam: float
    dtype: str                          # "fp32" | "bf16"
    seed: int = 0

    @property
    def seq_len(self) -> int:
        t, h, w = self.grid
        return t * h * w + self.text_tokens

    @property
    def num_blocks(self) -> int:
        return -(-self.seq_len // self.block)

    @property
    def keep_k(self) -> int:
        return keep_from_sparsity(self.num_blocks, self.sparsity)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # small case the fp64 oracle finishes in seconds
    "tiny-fp32": Workload("tiny-fp32", 1, 2, (16, 8, 8), 0, 64, 64, 0.75, 0.5, "fp32"),
    # image DiT: 64x64 latent + 512 text tokens
    "image-dit": Workload("image-dit", 1, 24, (1, 64, 64), 512, 128, 64, 0.75, 0.5, "bf16"),
    # video DiT, small: 21x30x52 latent grid
    "video-dit-small": Workload("video-dit-small", 1, 12, (21, 30, 52), 0, 128, 64, 0.875, 0.5, "bf16"),
    # video DiT, large: 21x45x80 latent grid, block 128
    "video-dit-large": Workload("video-dit-large", 1, 40, (21, 45, 80), 0, 128, 128, 0.875, 0.5, "bf16"),
}
# sequence-length / sparsity sweep (heads 16, d 128, block 64)
for _grid in [(8, 32, 32), (32, 32, 32), (32, 64, 64)]:
    for _sp in [0.5, 0.75, 0.875, 0.9375, 0.0]:
        _L = _grid[0] * _grid[1] * _grid[2]
        _n = f"sweep-L{_L}-s{_sp:g}"
        WORKLOADS[_n] = Workload(_n, 1, 16, _grid, 0, 128, 64, _sp, 0.5, "bf16")


def _field(rng: np.random.Generator, grid: Tuple[int, int, int], d: int) -> np.ndarray:
    T, Hg, W = grid
    omega = rng.uniform(0.5, 4.0, size=(4, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(4, d))
    amp = rng.standard_normal(size=(4, d))
    t = np.arange(T, dtype=np.float64) / T
    y = np.arange(Hg, dtype=np.float64) / Hg
    x = np.arange(W, dtype=np.float64) / W
    # phase of each sinusoid at each token, raster order (t, y, x)
    theta = (omega[:, 0, None, None, None] * t[None, :, None, None]
             + omega[:, 1, None, None, None] * y[None, None, :, None]
             + omega[:, 2, None, None, None] * x[None, None, None, :])
    theta = (2.0 * math.pi) * theta.reshape(4, -1)                     # [4, Limg]
    # sin(theta + phi) = sin(theta) cos(phi) + cos(theta) sin(phi): one [Limg x 8] @ [8 x d] product
    basis = np.concatenate([np.sin(theta), np.cos(theta)], axis=0).T   # [Limg, 8]
    coef = np.concatenate([amp * np.cos(phi), amp * np.sin(phi)], axis=0)  # [8, d]
    return (basis @ coef) * (2.0 ** -0.5)


def make_head(w: Workload, b: int, h: int, seed: Optional[int] = None):
    """float32 numpy arrays (q, k, v), each [L, d], for one (batch, head), before the dtype cast."""
    s = w.seed if seed is None else seed
    rng = np.random.default_rng([s, b, h])
    d = w.head_dim
    F = _field(rng, w.grid, d)
    n_img = F.shape[0]
    L = w.seq_len
    eq = rng.standard_normal(size=(L, d), dtype=np.float32)
    ek = rng.standard_normal(size=(L, d), dtype=np.float32)
    v = rng.standard_normal(size=(L, d), dtype=np.float32)
    q = eq.copy()
    k = ek.copy()
    q[:n_img] += (0.5 * F).astype(np.float32)
    k[:n_img] += (0.5 * F).astype(np.float32)
    q *= np.float32(1.0 / math.sqrt(d))
    return q, k, v


def to_dtype(x: np.ndarray, dtype: str):
    """Cast a float32 array to a CPU torch tensor of the run's dtype (round to nearest even)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)


def make_qkv(w: Workload, heads: Optional[Sequence[int]] = None, seed: Optional[int] = None):
    """CPU torch tensors q, k, v of shape [B, len(heads), L, d] in the workload's dtype.

    ``heads`` selects a subset of the workload's heads (default: all); head h always gets the same
    values whatever subset it is drawn in, so sampled checks see the full-size run's inputs.
    """
    import os
    from concurrent.futures import ThreadPoolExecutor

    import torch
    hs = list(range(w.heads)) if heads is None else list(heads)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    L, d = w.seq_len, w.head_dim
    out = [torch.empty((w.batch, len(hs), L, d), dtype=tdt) for _ in range(3)]

    def fill(bi):
        b, i = bi
        for t, arr in zip(out, make_head(w, b, hs[i], seed)):
            t[b, i].copy_(to_dtype(arr, w.dtype))

    # every (batch, head) draws from its own stream, so filling them on threads gives the same values
    jobs = [(b, i) for b in range(w.batch) for i in range(len(hs))]
    workers = min(len(jobs), os.cpu_count() or 1, 16)
    if workers <= 1:
        for job in jobs:
            fill(job)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, jobs))
    return out[0], out[1], out[2]


def make_block_structured(seq_len: int, head_dim: int, block: int, dtype: str, seed: int = 0,
                          spread: float = 0.5, qscale: float = 1.5):
    """CPU torch tensors q, k, v [1, 1, L, d] whose key blocks carry strong, block-specific
    key/value covariance, so that each block's first-order matrix differs markedly from their mean.

    From ``default_rng([seed, 1000003])``: per block j a centre c_j ~ 0.6 N(0,1)^d and a sign
    s_j in {-1, +1}; per token n of block j a deviation e_n ~ N(0,1)^d; then
        k_n = c_j + spread * e_n,    v_n = 0.5 N(0,1)^d + s_j * e_n,    q_n = qscale * N(0,1)^d / sqrt(d).
    """
    rng = np.random.default_rng([seed, 1000003])
    L, d = seq_len, head_dim
    nb = -(-L // block)
    centre = 0.6 * rng.standard_normal((nb, d))
    sign = rng.choice([-1.0, 1.0], size=nb)
    dev = rng.standard_normal((L, d))
    owner = np.arange(L) // block
    k = centre[owner] + spread * dev
    v = 0.5 * rng.standard_normal((L, d)) + sign[owner][:, None] * dev
    q = qscale * rng.standard_normal((L, d)) / math.sqrt(d)
    return tuple(to_dtype(x.astype(np.float32), dtype)[None, None] for x in (q, k, v))
