"""ctypes binding of the PISA C ABI (include/pisa.h): argument marshalling only.

Every step of the computation runs in the CUDA library ``lib/libpisa_b200.so``; torch supplies
device memory and the current stream.  There is no fallback: if the library is missing or fails to
load, every entry point raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libpisa_b200.so")

PISA_OK, PISA_ERR_INVALID_ARG, PISA_ERR_UNSUPPORTED, PISA_ERR_CUDA, PISA_ERR_DEVICE_TIMEOUT = range(5)
PISA_BF16, PISA_FP32, PISA_BF16_FP8QK = 0, 1, 2
PISA_MODE_PISA, PISA_MODE_EXACT_ONLY, PISA_MODE_PER_BLOCK = 0, 1, 2
PISA_DEVERR_WAIT_TIMEOUT, PISA_DEVERR_BAD_SELECTION = 1, 2

SYMBOLS = ("pisa_abi_version", "pisa_num_blocks", "pisa_stats_bytes", "pisa_stats_carve", "pisa_workspace_bytes",
           "pisa_precompute", "pisa_route", "pisa_attention", "pisa_read_device_error", "pisa_status_string",
           "pisa_precompute_noalloc", "pisa_testing_set_attention_fault", "pisa_perblock_workspace_bytes",
           "pisa_permute_rows", "pisa_axis_permutation", "pisa_precompute_zeroth_order", "pisa_precompute_route",
           "pisa_testing_set_precompute_fault")


class PisaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class PisaStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("qbar", "kbar", "vsum", "hbar", "M", "H", "kbar_op", "vsum_op", "hbar_op", "v_op", "vscale",
                 "hdiff_op", "q8", "k8", "kbar8", "qscale", "kscale", "kbscale")]


class PisaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"PISA CUDA library not built: {_LIB_PATH} is missing "
                               "(run python -m piecewise_approximate_attention_b200.build)")
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        sig = {
            "pisa_abi_version": (i32, []),
            "pisa_num_blocks": (i32, [i32, i32]),
            "pisa_stats_bytes": (sz, [P(PisaShape), i32]),
            "pisa_stats_carve": (i32, [P(PisaShape), vp, sz, i32, P(PisaStats)]),
            "pisa_workspace_bytes": (sz, [P(PisaShape)]),
            "pisa_perblock_workspace_bytes": (sz, [P(PisaShape)]),
            "pisa_precompute": (i32, [P(PisaShape), vp, vp, vp, P(PisaStats), vp, sz, vp]),
            "pisa_precompute_zeroth_order": (i32, [P(PisaShape), vp, vp, vp, P(PisaStats), vp, sz, vp]),
            "pisa_route": (i32, [P(PisaShape), P(PisaStats), i32, f32, vp, vp, vp, vp]),
            "pisa_precompute_route": (i32, [P(PisaShape), vp, vp, vp, P(PisaStats), i32, f32, vp, vp, vp, vp, sz,
                                            i32, vp]),
            "pisa_attention": (i32, [P(PisaShape), vp, vp, vp, P(PisaStats), vp, vp, i32, i32, vp, vp, sz, vp]),
            "pisa_read_device_error": (i32, [vp, P(i32), vp]),
            "pisa_status_string": (ctypes.c_char_p, [i32]),
            "pisa_precompute_noalloc": (i32, [P(PisaShape), vp, vp, vp, P(PisaStats), vp]),
            "pisa_testing_set_attention_fault": (i32, [i32, ctypes.c_uint64]),
            "pisa_testing_set_precompute_fault": (i32, [i32, ctypes.c_uint64]),
            "pisa_permute_rows": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp]),
            "pisa_axis_permutation": (i32, [i32, i32, i32, i32, ctypes.c_char_p, P(i32), ctypes.c_int64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pisa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != PISA_OK:
        raise PisaError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


# ---------------------------------------------------------------------------------------------
# Thin wrappers with the ABI's names
# ---------------------------------------------------------------------------------------------
def make_shape(batch, heads, seq_len, head_dim, block, dtype, softmax_scale=1.0) -> PisaShape:
    dt = {"bf16": PISA_BF16, "fp32": PISA_FP32, "bf16_fp8qk": PISA_BF16_FP8QK}.get(dtype, dtype)
    return PisaShape(batch, heads, seq_len, head_dim, block, int(dt), float(softmax_scale))


def shape_of(q, block: int, softmax_scale: float = 1.0) -> PisaShape:
    import torch
    B, H, L, d = q.shape
    dt = PISA_BF16 if q.dtype == torch.bfloat16 else PISA_FP32
    return make_shape(B, H, L, d, block, dt, softmax_scale)


def pisa_num_blocks(seq_len: int, block: int) -> int:
    return int(lib().pisa_num_blocks(seq_len, block))


def pisa_stats_bytes(shape: PisaShape, with_H: bool = False) -> int:
    return int(lib().pisa_stats_bytes(ctypes.byref(shape), int(with_H)))


def pisa_workspace_bytes(shape: PisaShape) -> int:
    return int(lib().pisa_workspace_bytes(ctypes.byref(shape)))


@dataclasses.dataclass
class Stats:
    """Device statistics (views into one carved buffer) and the C struct pointing at them."""
    buf: object
    c: PisaStats
    qbar: object
    kbar: object
    vsum: object
    hbar: object
    M: object
    H: Optional[object]
    kbar_op: object
    vsum_op: object
    hbar_op: object
    v_op: object
    vscale: object
    hdiff_op: Optional[object]
    q8: Optional[object] = None          # e4m3 copies (uint8 views) and scales, PISA_BF16_FP8QK only
    k8: Optional[object] = None
    kbar8: Optional[object] = None
    qscale: Optional[object] = None
    kscale: Optional[object] = None
    kbscale: Optional[object] = None


def alloc_stats(shape: PisaShape, device, with_H: bool = False) -> Stats:
    import torch
    n = pisa_stats_bytes(shape, with_H)
    if n == 0:
        raise PisaError(PISA_ERR_INVALID_ARG, "pisa_stats_bytes")
    buf = torch.empty(n, dtype=torch.uint8, device=device)
    st = PisaStats()
    _check(lib().pisa_stats_carve(ctypes.byref(shape), buf.data_ptr(), n, int(with_H), ctypes.byref(st)),
           "pisa_stats_carve")
    B, H, d = shape.batch, shape.heads, shape.head_dim
    nb = pisa_num_blocks(shape.seq_len, shape.block)
    base = buf.data_ptr()

    def view(ptr, dtype, dims):
        if not ptr:
            return None
        numel = 1
        for x in dims:
            numel *= x
        off = ptr - base
        esz = torch.empty((), dtype=dtype).element_size()
        return buf[off:off + numel * esz].view(dtype).view(*dims)

    f32, bf, f16 = torch.float32, torch.bfloat16, torch.float16
    return Stats(buf, st, view(st.qbar, f32, (B, H, nb, d)), view(st.kbar, f32, (B, H, nb, d)),
                 view(st.vsum, f32, (B, H, nb, d)), view(st.hbar, f32, (B, H, d, d)), view(st.M, f32, (B, H, nb)),
                 view(st.H, f32, (B, H, nb, d, d)), view(st.kbar_op, bf, (B, H, nb, d)),
                 view(st.vsum_op, f16, (B, H, nb, d)), view(st.hbar_op, bf, (B, H, d, d)),
                 view(st.v_op, f16, (B, H, shape.seq_len, d)), view(st.vscale, f32, (B, H)),
                 view(st.hdiff_op, bf, (B, H, nb, d, d)), view(st.q8, torch.uint8, (B, H, shape.seq_len, d)),
                 view(st.k8, torch.uint8, (B, H, shape.seq_len, d)), view(st.kbar8, torch.uint8, (B, H, nb, d)),
                 view(st.qscale, f32, (B, H, shape.seq_len)), view(st.kscale, f32, (B, H, nb)),
                 view(st.kbscale, f32, (B, H, (nb + 127) // 128)))


def pisa_perblock_workspace_bytes(shape: PisaShape) -> int:
    return int(lib().pisa_perblock_workspace_bytes(ctypes.byref(shape)))


def alloc_workspace(shape: PisaShape, device, per_block: bool = False):
    """Zeroed device workspace (the status word must start at zero); per_block sizes it for
    PISA_MODE_PER_BLOCK."""
    import torch
    n = pisa_perblock_workspace_bytes(shape) if per_block else pisa_workspace_bytes(shape)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def pisa_precompute(shape: PisaShape, q, k, v, stats: Stats, ws, stream=None):
    _check(lib().pisa_precompute(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(stats.c), _ptr(ws),
                                 ws.numel(), _stream(stream)), "pisa_precompute")


def pisa_precompute_zeroth_order(shape: PisaShape, q, k, v, stats: Stats, ws, stream=None):
    """Zeroth-order statistics only (what lambda = 0 routing and the keep-or-drop mode read)."""
    _check(lib().pisa_precompute_zeroth_order(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(stats.c),
                                              _ptr(ws), ws.numel(), _stream(stream)), "pisa_precompute_zeroth_order")


def pisa_precompute_noalloc(shape: PisaShape, q, k, v, stats: Stats, stream=None):
    """pisa_precompute with the library's fixed device scratch instead of a caller workspace."""
    _check(lib().pisa_precompute_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(stats.c),
                                         _stream(stream)), "pisa_precompute_noalloc")


def pisa_route(shape: PisaShape, stats: Stats, keep_k: int, lam: float, sel, order=None, scores=None, stream=None):
    _check(lib().pisa_route(ctypes.byref(shape), ctypes.byref(stats.c), int(keep_k), float(lam), _ptr(sel),
                            _ptr(order), _ptr(scores), _stream(stream)), "pisa_route")


PISA_PRECOMPUTE_ROUTE_FUSED = 1


def pisa_precompute_route(shape: PisaShape, q, k, v, stats: Stats, keep_k: int, lam: float, sel, order, scores, ws,
                          fused: bool = False, stream=None):
    """pisa_precompute then pisa_route; with fused, one cluster launch for bf16 inputs with nb <= 128."""
    _check(lib().pisa_precompute_route(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(stats.c),
                                       int(keep_k), float(lam), _ptr(sel), _ptr(order), _ptr(scores), _ptr(ws),
                                       ws.numel(), PISA_PRECOMPUTE_ROUTE_FUSED if fused else 0, _stream(stream)),
           "pisa_precompute_route")


def pisa_attention(shape: PisaShape, q, k, v, stats: Stats, sel, order, keep_k: int, mode: int, o, ws, stream=None):
    _check(lib().pisa_attention(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(stats.c), _ptr(sel),
                                _ptr(order), int(keep_k), int(mode), _ptr(o), _ptr(ws), ws.numel(), _stream(stream)),
           "pisa_attention")


def pisa_permute_rows(src, dst, perm, inverse: bool = False, stream=None):
    """Rows of src [..., L, row] into dst through perm ([L] shared, or one row of perm per head)."""
    L = src.shape[-2]
    bh = src.numel() // (L * src.shape[-1])
    row_bytes = src.shape[-1] * src.element_size()
    per_head = 1 if perm.dim() > 1 else 0
    _check(lib().pisa_permute_rows(_ptr(src), _ptr(dst), _ptr(perm), bh, L, row_bytes, per_head, int(bool(inverse)),
                                   _stream(stream)), "pisa_permute_rows")


def pisa_axis_permutation(grid, order: str, extra_tokens: int = 0):
    """Host int32 numpy permutation of a (frames, height, width) raster grid listed in `order`."""
    import numpy as np
    T, Hg, W = grid
    out = np.empty(T * Hg * W + extra_tokens, dtype=np.int32)
    _check(lib().pisa_axis_permutation(T, Hg, W, extra_tokens, order.encode(),
                                       out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), out.size),
           "pisa_axis_permutation")
    return out


def pisa_read_device_error(ws, stream=None):
    """(status, code) of the workspace's device status word; clears it."""
    code = ctypes.c_int32(0)
    st = lib().pisa_read_device_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    return int(st), int(code.value)
