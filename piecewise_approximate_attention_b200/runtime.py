"""Buffers and call sequence for one PISA attention shape (pre-compute -> route -> attention).

All three steps run in the CUDA library through the C ABI; this module only allocates device
memory with torch and passes pointers and the current stream.
"""
from __future__ import annotations

from typing import Optional

from . import _lib as C


class Pisa:
    """Reusable PISA attention for a fixed [B, H, L, d] shape, block size, keep_k and lambda.

    ``pair=True`` asks the router for the query-block pairing order used by 128-row tiles when
    block == 64 (a scheduling choice: the output does not depend on it).  ``first_order=False``
    makes ``precompute`` write the zeroth-order statistics only (pisa_precompute_zeroth_order):
    enough for lambda = 0 routing and the keep-or-drop mode, i.e. an exact-only pipeline.
    """

    def __init__(self, batch: int, heads: int, seq_len: int, head_dim: int, block: int, keep_k: int,
                 lam: float, dtype: str = "bf16", softmax_scale: float = 1.0, device="cuda",
                 mode: int = C.PISA_MODE_PISA, with_H: bool = False, pair: bool = True,
                 first_order: bool = True):
        import torch
        if not first_order and (lam != 0.0 or mode != C.PISA_MODE_EXACT_ONLY):
            raise ValueError("the zeroth-order statistics serve lambda = 0 routing and PISA_MODE_EXACT_ONLY only")
        self.first_order = first_order
        self.shape = C.make_shape(batch, heads, seq_len, head_dim, block, dtype, softmax_scale)
        self.block, self.keep_k, self.lam, self.mode = block, keep_k, lam, mode
        self.nb = C.pisa_num_blocks(seq_len, block)
        self.device = torch.device(device)
        self.tdtype = torch.float32 if dtype == "fp32" else torch.bfloat16
        self.fp8 = dtype == "bf16_fp8qk"
        self._torch_f32 = torch.float32
        if mode == C.PISA_MODE_PER_BLOCK:
            with_H = True         # the per-block first-order matrices live in the stats
        self.stats = C.alloc_stats(self.shape, self.device, with_H)
        self.ws = C.alloc_workspace(self.shape, self.device, per_block=mode == C.PISA_MODE_PER_BLOCK)
        self.sel = torch.empty((batch, heads, self.nb, max(keep_k, 1)), dtype=torch.int32, device=self.device)
        self.order = torch.empty((batch, heads, self.nb), dtype=torch.int32, device=self.device) if pair else None

    def precompute(self, q, k, v, stream=None):
        if self.first_order:
            C.pisa_precompute(self.shape, q, k, v, self.stats, self.ws, stream)
        else:
            C.pisa_precompute_zeroth_order(self.shape, q, k, v, self.stats, self.ws, stream)

    def fused_short_step(self) -> bool:
        """Whether precompute_route(fused=True) is one cluster launch (bf16 inputs, head_dim 128,
        nb <= 128; the device must also fit every head's cluster at once)."""
        return self.first_order and self.tdtype != self._torch_f32 and self.shape.head_dim == 128 and self.nb <= 128

    def precompute_route(self, q, k, v, scores=None, stream=None, fused: bool = False):
        """Pre-computation and routing through pisa_precompute_route: the separate kernels, or with
        ``fused`` (short sequences) one cluster launch; the results are the same either way."""
        if not self.first_order:
            self.precompute(q, k, v, stream)
            self.route(scores, stream)
            return
        C.pisa_precompute_route(self.shape, q, k, v, self.stats, self.keep_k, self.lam, self.sel, self.order, scores,
                                self.ws, fused, stream)

    def route(self, scores=None, stream=None):
        C.pisa_route(self.shape, self.stats, self.keep_k, self.lam, self.sel, self.order, scores, stream)

    def attention(self, q, k, v, o, sel=None, order=None, mode: Optional[int] = None, stream=None):
        s = self.sel if sel is None else sel
        od = self.order if order is None else order
        C.pisa_attention(self.shape, q, k, v, self.stats, s, od, self.keep_k, self.mode if mode is None else mode,
                         o, self.ws, stream)

    def __call__(self, q, k, v, o=None, stream=None):
        import torch
        if o is None:
            o = torch.empty_like(q)
        self.precompute_route(q, k, v, stream=stream)
        self.attention(q, k, v, o, stream=stream)
        return o

    def capture(self, q, k, v, o, fused: bool = False):
        """Records one full step (pre-computation, routing, attention of q, k, v into o) as a CUDA
        graph and returns it; ``graph.replay()`` then re-runs the step on whatever the same
        buffers hold, with one launch from the host.  The buffers must stay allocated while the
        graph is used.  The step runs once eagerly first (outside the capture).  ``fused=True``
        records the fused pre-computation and routing (short sequences) instead of the separate
        calls."""
        import torch
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            self(q, k, v, o)
        torch.cuda.current_stream(self.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.precompute_route(q, k, v, fused=fused)
            self.attention(q, k, v, o)
        return graph

    def launches_per_step(self) -> int:
        """Kernels one __call__ enqueues: pre-compute 3 (2 zeroth-order only on the bf16 path, 1 on
        the fp32 path; +3 e4m3 quantizations), routing 1 (+1 pairing), attention 1 (+1 for the
        per-block first-order kernel on the bf16 path)."""
        extra = 1 if (self.mode == C.PISA_MODE_PER_BLOCK and self.tdtype != self._torch_f32 and
                      self.keep_k < self.nb) else 0
        pre = 3 if self.first_order else (1 if self.tdtype == self._torch_f32 else 2)
        route = 1 + (1 if self.order is not None else 0)
        return pre + (3 if self.fp8 else 0) + route + 1 + extra

    def device_error(self, stream=None):
        return C.pisa_read_device_error(self.ws, stream)


AXIS_ORDERS = ("thw", "twh", "htw", "hwt", "wth", "wht")


def reorder_tokens(x, perm, out=None, stream=None):
    """x [B, H, L, d] with its rows gathered through perm ([L], or [B*H, L] per head) on the GPU."""
    import torch
    out = torch.empty_like(x) if out is None else out
    C.pisa_permute_rows(x, out, perm, inverse=False, stream=stream)
    return out


def restore_tokens(x, perm, out=None, stream=None):
    """Inverse of reorder_tokens: rows of x scattered back to their original positions."""
    import torch
    out = torch.empty_like(x) if out is None else out
    C.pisa_permute_rows(x, out, perm, inverse=True, stream=stream)
    return out


def axis_order_permutations(grid, extra_tokens: int = 0, device="cuda"):
    """Device int32 permutations [6, L] for the six axis orders of a (frames, height, width) grid."""
    import torch
    return torch.stack([torch.from_numpy(C.pisa_axis_permutation(grid, o, extra_tokens)) for o in AXIS_ORDERS]).to(device)


def choose_axis_order(pisa: "Pisa", q, k, v, perms):
    """Per head, the axis order whose blocks have the smallest total first-order spread sum_j M_j
    (the method's own covariance measure, from the pre-computation on the reordered tokens).
    Returns (per-head permutation [B*H, L] int32, chosen order index per head).  A calibration
    step: six pre-computations."""
    import torch
    B, H = q.shape[0], q.shape[1]
    scores = []
    for r in range(perms.shape[0]):
        qq, kk, vv = (reorder_tokens(x, perms[r]) for x in (q, k, v))
        pisa.precompute(qq, kk, vv)
        scores.append(pisa.stats.M.reshape(B * H, -1).sum(dim=1))
    best = torch.stack(scores).argmin(dim=0)
    return perms[best].contiguous(), best


class HostPipeline:
    """Steps whose inputs and outputs live in (pinned) host memory, with the copies overlapped:
    the inputs of step i+1 are uploaded and the output of step i-1 is downloaded while step i
    runs.  Two device buffer sets and three streams (upload, compute, download), ordered by
    events; the statistics and routing buffers of `pisa` are reused by consecutive steps on the
    compute stream.  ``submit`` only enqueues; ``synchronize`` waits for everything submitted."""

    def __init__(self, pisa: "Pisa", q_like):
        import torch
        self.p = pisa
        dev = pisa.device
        self.bufs = [[torch.empty(q_like.shape, dtype=q_like.dtype, device=dev) for _ in range(4)] for _ in range(2)]
        self.s_in, self.s_cmp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_cmp = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.i = 0

    def submit(self, qh, kh, vh, oh):
        import torch
        b = self.i % 2
        q, k, v, o = self.bufs[b]
        with torch.cuda.stream(self.s_in):
            self.s_in.wait_event(self.ev_cmp[b])          # step i-2 has finished reading q, k, v
            q.copy_(qh, non_blocking=True)
            k.copy_(kh, non_blocking=True)
            v.copy_(vh, non_blocking=True)
            self.ev_in[b].record(self.s_in)
        with torch.cuda.stream(self.s_cmp):
            self.s_cmp.wait_event(self.ev_in[b])
            self.s_cmp.wait_event(self.ev_out[b])         # the download of step i-2 has read o
            self.p.precompute(q, k, v, stream=self.s_cmp)
            self.p.route(stream=self.s_cmp)
            self.p.attention(q, k, v, o, stream=self.s_cmp)
            self.ev_cmp[b].record(self.s_cmp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.ev_cmp[b])
            oh.copy_(o, non_blocking=True)
            self.ev_out[b].record(self.s_out)
        self.i += 1

    def synchronize(self):
        for s in (self.s_in, self.s_cmp, self.s_out):
            s.synchronize()
