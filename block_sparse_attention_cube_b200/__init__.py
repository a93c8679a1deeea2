"""B200 (sm_100a) cube-based Video Sparse Attention and dense attention.

Thin Python binding over the C ABI in include/vsa.h: each function checks
dtypes and contiguity, allocates outputs with torch (device memory is the
only thing torch provides here), and calls the library on the current CUDA
stream.  Every step of the computation runs in the library's kernels.

Layouts (see include/vsa.h): q/k/v/out are [B, N, H, D] bf16 with token
n = (t*X + x)*Y + y; tiled tensors are [B, H, Npad, D] bf16, cube-major.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _lib

_L = _lib.load()


class VsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_lib.STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


@dataclass(frozen=True)
class Shape:
    batch: int
    heads: int
    head_dim: int
    grid: Tuple[int, int, int]   # (T, X, Y) tokens

    def c(self) -> _lib.VsaShape:
        t, x, y = self.grid
        return _lib.VsaShape(self.batch, self.heads, self.head_dim, t, x, y)

    @property
    def tokens(self) -> int:
        t, x, y = self.grid
        return t * x * y


def _check(st: int) -> None:
    if st != _lib.VSA_OK:
        raise VsaError(st, _L.vsa_last_error().decode(errors="replace"))


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor], dtype: torch.dtype, name: str) -> Optional[int]:
    if t is None:
        return None
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def abi_version() -> int:
    return int(_L.vsa_abi_version())


def shape_info(shape: Shape) -> Tuple[int, int]:
    """(Npad, C) of a shape."""
    npad, c = ctypes.c_int64(), ctypes.c_int32()
    _check(_L.vsa_shape_info(ctypes.byref(shape.c()), ctypes.byref(npad), ctypes.byref(c)))
    return int(npad.value), int(c.value)


def default_scale(shape: Shape) -> float:
    return 1.0 / math.sqrt(shape.head_dim)


def tile(x: torch.Tensor, shape: Shape, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    npad, _ = shape_info(shape)
    if out is None:
        out = torch.empty((shape.batch, shape.heads, npad, shape.head_dim), dtype=torch.bfloat16, device=x.device)
    _check(_L.vsa_tile(ctypes.byref(shape.c()), _ptr(x, torch.bfloat16, "x"), _ptr(out, torch.bfloat16, "xt"),
                       _stream()))
    return out


def untile(xt: torch.Tensor, shape: Shape, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    if out is None:
        out = torch.empty((shape.batch, shape.tokens, shape.heads, shape.head_dim), dtype=torch.bfloat16,
                          device=xt.device)
    _check(_L.vsa_untile(ctypes.byref(shape.c()), _ptr(xt, torch.bfloat16, "xt"), _ptr(out, torch.bfloat16, "x"),
                         _stream()))
    return out


def pool(xt: torch.Tensor, shape: Shape) -> torch.Tensor:
    _, c = shape_info(shape)
    out = torch.empty((shape.batch, shape.heads, c, shape.head_dim), dtype=torch.float32, device=xt.device)
    _check(_L.vsa_pool(ctypes.byref(shape.c()), _ptr(xt, torch.bfloat16, "xt"), _ptr(out, torch.float32, "xbar"),
                       _stream()))
    return out


def coarse(qbar: torch.Tensor, kbar: torch.Tensor, vbar: torch.Tensor, shape: Shape,
           scale: Optional[float] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    _, c = shape_info(shape)
    scale = default_scale(shape) if scale is None else scale
    scores = torch.empty((shape.batch, shape.heads, c, c), dtype=torch.float32, device=qbar.device)
    oc = torch.empty_like(qbar)
    n = int(_L.vsa_coarse_workspace_bytes(ctypes.byref(shape.c())))
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=qbar.device)
    _check(_L.vsa_coarse(ctypes.byref(shape.c()), _ptr(qbar, torch.float32, "qbar"), _ptr(kbar, torch.float32, "kbar"),
                         _ptr(vbar, torch.float32, "vbar"), scale, _ptr(scores, torch.float32, "scores"),
                         _ptr(oc, torch.float32, "o_coarse"), _ptr(ws, torch.uint8, "workspace"), ws.numel(),
                         _stream()))
    return scores, oc


def topk(scores: torch.Tensor, shape: Shape, k: int) -> torch.Tensor:
    _, c = shape_info(shape)
    idx = torch.empty((shape.batch, shape.heads, c, k), dtype=torch.int32, device=scores.device)
    _check(_L.vsa_topk(ctypes.byref(shape.c()), _ptr(scores, torch.float32, "scores"), k,
                       _ptr(idx, torch.int32, "idx"), _stream()))
    return idx


def group(scores: torch.Tensor, shape: Shape) -> torch.Tensor:
    """Work order for fine(): per head, query cubes with similar selections next to each other."""
    _, c = shape_info(shape)
    order = torch.empty((shape.batch, shape.heads, c), dtype=torch.int32, device=scores.device)
    _check(_L.vsa_group(ctypes.byref(shape.c()), _ptr(scores, torch.float32, "scores"),
                        _ptr(order, torch.int32, "order"), _stream()))
    return order


def fine(qt: torch.Tensor, kt: torch.Tensor, vt: torch.Tensor, shape: Shape, idx: Optional[torch.Tensor] = None,
         scale: Optional[float] = None, want_lse: bool = True,
         order: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Fine attention over the selected cubes (idx [B,H,C,k] int32, or None for all cubes).

    `order` ([B,H,C] int32 permutation, e.g. from group()) sets the work order only.
    """
    scale = default_scale(shape) if scale is None else scale
    k = int(idx.shape[-1]) if idx is not None else 0
    o = torch.empty_like(qt)
    lse = torch.empty(qt.shape[:3], dtype=torch.float32, device=qt.device) if want_lse else None
    _check(_L.vsa_fine(ctypes.byref(shape.c()), _ptr(qt, torch.bfloat16, "qt"), _ptr(kt, torch.bfloat16, "kt"),
                       _ptr(vt, torch.bfloat16, "vt"), _ptr(idx, torch.int32, "idx"), k,
                       _ptr(order, torch.int32, "order"), scale,
                       _ptr(o, torch.bfloat16, "o_fine"), _ptr(lse, torch.float32, "lse"), _stream()))
    return o, lse


def combine(o_coarse: torch.Tensor, o_fine: torch.Tensor, shape: Shape, g_coarse: Optional[torch.Tensor] = None,
            g_fine: Optional[torch.Tensor] = None) -> torch.Tensor:
    out = torch.empty_like(o_fine)
    _check(_L.vsa_combine(ctypes.byref(shape.c()), _ptr(o_coarse, torch.float32, "o_coarse"),
                          _ptr(o_fine, torch.bfloat16, "o_fine"), _ptr(g_coarse, torch.bfloat16, "g_coarse"),
                          _ptr(g_fine, torch.bfloat16, "g_fine"), _ptr(out, torch.bfloat16, "o_tiled"), _stream()))
    return out


def topk_order(scores: torch.Tensor, shape: Shape, k: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """topk() and group() from one pass over the scores (C <= 2048): (idx [B,H,C,k], order [B,H,C])."""
    _, c = shape_info(shape)
    idx = torch.empty((shape.batch, shape.heads, c, k), dtype=torch.int32, device=scores.device)
    order = torch.empty((shape.batch, shape.heads, c), dtype=torch.int32, device=scores.device)
    sig = torch.empty((shape.batch, shape.heads, c), dtype=torch.int64, device=scores.device)
    _check(_L.vsa_topk_order(ctypes.byref(shape.c()), _ptr(scores, torch.float32, "scores"), k,
                             _ptr(idx, torch.int32, "idx"), _ptr(order, torch.int32, "order"),
                             _ptr(sig, torch.int64, "sig_scratch"), _stream()))
    return idx, order


def pool_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             shape: Shape) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Cube means of q, k, v ([B,N,H,D] token layout) in one launch: three [B,H,C,D] float32 tensors."""
    _, c = shape_info(shape)
    outs = [torch.empty((shape.batch, shape.heads, c, shape.head_dim), dtype=torch.float32, device=q.device)
            for _ in range(3)]
    _check(_L.vsa_pool_qkv(ctypes.byref(shape.c()), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                           _ptr(v, torch.bfloat16, "v"), *(_ptr(o, torch.float32, n) for o, n in
                                                            zip(outs, ("qbar", "kbar", "vbar"))), _stream()))
    return outs[0], outs[1], outs[2]


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, shape: Shape, w_q: Optional[torch.Tensor] = None,
                 w_k: Optional[torch.Tensor] = None, eps: float = 1e-6, theta: float = 10000.0,
                 token_offset: int = 0, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                 inplace: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Q/K RMSNorm over H*D then 3D RoPE of [B, n, H, D] rows of global tokens token_offset..+n-1.

    Returns (q_out, k_out): new tensors, the given `out` pair, or q and k themselves when `inplace`."""
    n = int(q.shape[1])
    if inplace:
        qo, ko = q, k
    elif out is not None:
        qo, ko = out
    else:
        qo, ko = torch.empty_like(q), torch.empty_like(k)
    _check(_L.vsa_qk_norm_rope(ctypes.byref(shape.c()), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                               _ptr(w_q, torch.bfloat16, "w_q"), _ptr(w_k, torch.bfloat16, "w_k"), eps, theta,
                               token_offset, n, _ptr(qo, torch.bfloat16, "q_out"), _ptr(ko, torch.bfloat16, "k_out"),
                               _stream()))
    return qo, ko


def schedule(idx: torch.Tensor, shape: Shape, order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Precomputed steps of the fine stage for the selection idx [B,H,C,k] (and work order)."""
    k = int(idx.shape[-1])
    n = int(_L.vsa_schedule_bytes(ctypes.byref(shape.c()), k))
    steps = torch.empty(max(n, 1), dtype=torch.uint8, device=idx.device)
    _check(_L.vsa_schedule(ctypes.byref(shape.c()), _ptr(idx, torch.int32, "idx"), k,
                           _ptr(order, torch.int32, "order"), _ptr(steps, torch.uint8, "steps"), _stream()))
    return steps


def fine_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shape: Shape, idx: Optional[torch.Tensor] = None,
               scale: Optional[float] = None, order: Optional[torch.Tensor] = None,
               o_coarse: Optional[torch.Tensor] = None, g_coarse: Optional[torch.Tensor] = None,
               g_fine: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
               steps: Optional[torch.Tensor] = None, overflow: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Fine attention + gated merge on the token layout, written as [B,N,H,D] (idx None: dense attention).

    `steps` (from schedule()) replaces the kernel's own walk of the selection; the fixed-maximum
    kernel that then runs (and runs for dense attention) reports an overflow (and the re-run it
    caused) in `overflow`, int32 on the device with at least two elements: [0] the overflow word,
    [1] the kernel's work counter (allocated here when omitted)."""
    scale = default_scale(shape) if scale is None else scale
    kk = int(idx.shape[-1]) if idx is not None else 0
    if out is None:
        out = torch.empty_like(q)
    fixed_max = steps is not None or idx is None   # the one-tile kernel: sparse with steps, and dense
    if fixed_max and overflow is None:
        overflow = torch.empty(4, dtype=torch.int32, device=q.device)
    if fixed_max and overflow.numel() < 2:
        raise ValueError("overflow needs two int32 elements (the overflow word and the work counter)")
    _check(_L.vsa_fine_fused(ctypes.byref(shape.c()), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                             _ptr(v, torch.bfloat16, "v"), _ptr(idx, torch.int32, "idx"), kk,
                             _ptr(order, torch.int32, "order"), _ptr(steps, torch.uint8, "steps"), scale,
                             _ptr(o_coarse, torch.float32, "o_coarse"), _ptr(g_coarse, torch.bfloat16, "g_coarse"),
                             _ptr(g_fine, torch.bfloat16, "g_fine"), _ptr(out, torch.bfloat16, "out"),
                             _ptr(overflow, torch.int32, "overflow"), _stream()))
    return out


def forward_rerun(shape: Shape, topk_k: int, workspace: torch.Tensor, has_g_coarse: bool) -> bool:
    """After forward() on `workspace`: did its fixed-maximum fine stage overflow and re-run (synchronizes)?"""
    r = ctypes.c_int32(-1)
    _check(_L.vsa_forward_rerun(ctypes.byref(shape.c()), topk_k, int(bool(has_g_coarse)),
                                _ptr(workspace, torch.uint8, "workspace"), ctypes.byref(r), _stream()))
    return bool(r.value)


def workspace_bytes(shape: Shape, k: int) -> int:
    return int(_L.vsa_workspace_bytes(ctypes.byref(shape.c()), k))


def workspace_bytes_host(shape: Shape, k: int) -> int:
    return int(_L.vsa_workspace_bytes_host(ctypes.byref(shape.c()), k))


def alloc_workspace(shape: Shape, k: int, host_io: bool = False, device=None) -> torch.Tensor:
    n = workspace_bytes_host(shape, k) if host_io else workspace_bytes(shape, k)
    if n == 0:
        raise VsaError(1, "invalid shape or top-k for the workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shape: Shape, topk_k: int,
            scale: Optional[float] = None, g_coarse: Optional[torch.Tensor] = None,
            g_fine: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole VSA call: pool_qkv -> coarse -> topk_order -> schedule -> fine_fused (topk_k == C: dense fine stage)."""
    scale = default_scale(shape) if scale is None else scale
    if workspace is None:
        workspace = alloc_workspace(shape, topk_k, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(_L.vsa_forward(ctypes.byref(shape.c()), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                          _ptr(v, torch.bfloat16, "v"), _ptr(g_coarse, torch.bfloat16, "g_coarse"),
                          _ptr(g_fine, torch.bfloat16, "g_fine"), topk_k, scale,
                          _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                          _ptr(out, torch.bfloat16, "out"), _stream()))
    return out


def forward_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shape: Shape, topk_k: int,
                    scale: Optional[float] = None, g_coarse: Optional[torch.Tensor] = None,
                    g_fine: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """vsa_forward_noalloc: the whole call on the library's static device workspace.

    For callers that cannot allocate device memory (see include/vsa.h); the
    output buffer is still the caller's (allocated here only when omitted).
    Shapes whose workspace exceeds VSA_NOALLOC_WORKSPACE_BYTES raise VsaError.
    """
    scale = default_scale(shape) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    _check(_L.vsa_forward_noalloc(ctypes.byref(shape.c()), _ptr(q, torch.bfloat16, "q"),
                                  _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
                                  _ptr(g_coarse, torch.bfloat16, "g_coarse"), _ptr(g_fine, torch.bfloat16, "g_fine"),
                                  topk_k, scale, _ptr(out, torch.bfloat16, "out"), _stream()))
    return out


NOALLOC_WORKSPACE_BYTES = 32 << 20


def _host_ptr(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CPU tensor (pinned for asynchronous copies)")
    return t.data_ptr()


def forward_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shape: Shape, topk_k: int,
                 workspace: torch.Tensor, out: torch.Tensor, scale: Optional[float] = None,
                 g_coarse: Optional[torch.Tensor] = None, g_fine: Optional[torch.Tensor] = None) -> torch.Tensor:
    """vsa_forward_host: host tensors in and out. With two or more heads the copies run by head groups on
    the library's two copy streams, overlapping the compute on the current stream, which waits for the
    last copy; `out` is valid once the current stream is synchronized. Pin the host tensors for overlap."""
    scale = default_scale(shape) if scale is None else scale
    _check(_L.vsa_forward_host(ctypes.byref(shape.c()), _host_ptr(q, "q"), _host_ptr(k, "k"), _host_ptr(v, "v"),
                               _host_ptr(g_coarse, "g_coarse"), _host_ptr(g_fine, "g_fine"), topk_k, scale,
                               _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                               _host_ptr(out, "out"), _stream()))
    return out


def device_status() -> None:
    """Synchronize the current stream and raise VsaError if a device-side wait gave up."""
    _check(_L.vsa_device_status(_stream()))


def debug_wait_probe(limit_ns: int) -> None:
    _check(_L.vsa_debug_wait_probe(int(limit_ns), _stream()))


def raw_call(name: str, *args) -> int:
    """Call a C entry point directly and return its status (tests of argument checking)."""
    return int(getattr(_L, name)(*args))


def last_error() -> str:
    return _L.vsa_last_error().decode(errors="replace")
