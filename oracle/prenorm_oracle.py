"""Plain fp64 CPU oracle for the pre-attention pass: Q/K RMSNorm + 3D RoPE.

TEST INFRASTRUCTURE ONLY.  The parity tests and the benchmark's CPU-baseline
leg call this module for expected values.  The product path (the CUDA library
and its Python binding) never imports, links or runs anything here, and this
module imports nothing from it.

Sources.
* WorldFoundry inference-optimisation guide (openenvision.org, "推理优化"),
  table of exact or numerically equivalent Wan kernels, row "fused_rope": the
  3D rotary embedding of the native Wan DiT runs as one fused kernel; it works
  under Ulysses sequence parallelism, the kernel being told the rank's token
  offset and the padding; the rotation is evaluated in fp32 or fp64.
* Wan2.2 real-time inference teardown (zharfai.com), section "Fusion targets
  launch overhead and memory": after attention is fast, the Q/K normalisation
  (RMSNorm) shows up as many small kernels whose intermediates round-trip HBM;
  the fix reads each tensor once, runs the element-wise and reduction steps
  in registers, and writes once.

Readings where the pages leave a step open (both pages name the operations,
neither gives their formulas):
* RMSNorm runs over each token's whole projection vector (all H*D channels of
  Q, or of K), y = x / sqrt(mean(x^2) + eps) * w with a learned weight w of
  H*D values (w = 1 when absent) and eps = 1e-6 unless given;
* RoPE then rotates each head's channel pairs (2i, 2i+1), i < D/2.  The D/2
  pairs form three contiguous bands for the t, x and y axes, in that order;
  the x and y bands hold floor(D/6) pairs each and the t band the rest
  (22/21/21 pairs at D = 128, 12/10/10 at D = 64).  Pair j of a band of P
  pairs turns by angle pos * theta^(-j/P), pos being the token's coordinate
  on that band's axis, theta = 10000 unless given; the turn maps (a, b) to
  (a cos - b sin, a sin + b cos);
* a token's coordinates follow the token order n = (t*X + x)*Y + y;
* a call may cover one sequence-parallel shard: global tokens
  [token_offset, token_offset + n_tokens).  Global indices >= N are the
  padding that evens out the shards and come out as zero rows.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

DEFAULT_EPS = 1e-6
DEFAULT_THETA = 10000.0


def rope_bands(head_dim: int) -> Tuple[int, int, int]:
    """Rotation pairs per axis band (t, x, y) for one head of width head_dim."""
    assert head_dim % 2 == 0
    pairs = head_dim // 2
    p_xy = head_dim // 6
    return pairs - 2 * p_xy, p_xy, p_xy


def token_coords(n: np.ndarray, grid: Tuple[int, int, int]) -> np.ndarray:
    """(t, x, y) of global token indices n under n = (t*X + x)*Y + y; shape [len(n), 3]."""
    _, X, Y = grid
    n = np.asarray(n, dtype=np.int64)
    return np.stack([n // (X * Y), (n // Y) % X, n % Y], axis=-1)


def rope_angles(coords: np.ndarray, head_dim: int, theta: float = DEFAULT_THETA) -> np.ndarray:
    """Turn angle of every rotation pair: [len(coords), head_dim/2], float64."""
    coords = np.asarray(coords, dtype=np.float64)
    cols = []
    for axis, p in enumerate(rope_bands(head_dim)):
        freq = theta ** (-np.arange(p, dtype=np.float64) / p)
        cols.append(coords[:, axis:axis + 1] * freq[None, :])
    return np.concatenate(cols, axis=1)


def rope_apply(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate the channel pairs of x [n, H, D] by angles [n, D/2] (the same for every head)."""
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def rms_norm(x: np.ndarray, w: Optional[np.ndarray], eps: float = DEFAULT_EPS) -> np.ndarray:
    """RMSNorm of each row of x [..., C] over its C channels, times the weight w [C] (1 if None)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    return y if w is None else y * w


def norm_rope(x: np.ndarray, grid: Tuple[int, int, int], w: Optional[np.ndarray] = None,
              eps: float = DEFAULT_EPS, theta: float = DEFAULT_THETA, token_offset: int = 0) -> np.ndarray:
    """RMSNorm over H*D, then 3D RoPE, of one tensor x [B, n, H, D] (float64) whose row i is global
    token token_offset + i.  Rows past the grid's N tokens come out as zeros."""
    B, n, H, D = x.shape
    T, X, Y = grid
    N = T * X * Y
    g = token_offset + np.arange(n, dtype=np.int64)
    real = g < N
    out = np.zeros_like(x)
    if not real.any():
        return out
    y = rms_norm(x[:, real].reshape(B, -1, H * D), w, eps).reshape(B, -1, H, D)
    ang = rope_angles(token_coords(g[real], grid), D, theta)
    for b in range(B):
        out[b, real] = rope_apply(y[b], ang)
    return out


def qk_norm_rope(q: np.ndarray, k: np.ndarray, grid: Tuple[int, int, int], w_q: Optional[np.ndarray] = None,
                 w_k: Optional[np.ndarray] = None, eps: float = DEFAULT_EPS, theta: float = DEFAULT_THETA,
                 token_offset: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """The pre-attention pass on Q and K [B, n, H, D] (float64), exact."""
    return (norm_rope(q, grid, w_q, eps, theta, token_offset),
            norm_rope(k, grid, w_k, eps, theta, token_offset))
