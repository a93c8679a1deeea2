"""Seeded synthetic inputs for the video-DiT self-attention workloads.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle.  It holds the workload shapes and the random draws only: no step of
the attention method (no tiling, pooling, scoring, selection or softmax) is
computed here.

Workloads (token grid T x X x Y = frames x height x width tokens, token
n = (t*X + x)*Y + y, arrays laid out [B, N, H, D] as a DiT projects them,
``q_proj(x).view(b, s, heads, head_dim)`` in the Wan2.1 acceleration article
(bafh001.com), section 4.2):

* ``tiny_8x8x8``      1 x (8x8x8)    2 heads, d=64,  iid N(0,1), top-k 2 (and 8 = all)
* ``padded_7x15x16``  1 x (7x15x16)  4 heads, d=128, field inputs, top-k 8
* ``wan480p_dense``   1 x (21x30x52) 40 heads, d=128, field inputs, top-k = all 624 cubes
* ``wan480p_vsa_k32`` same data as ``wan480p_dense``, top-k 32
* ``wan720p_cfg_k64`` 2 x (21x45x80) 40 heads, d=128, field inputs, top-k 64

The 480p grid (21 latent frames of 30x52 patches, 40 heads of width 128) is
the workload of the Wan2.2 real-time inference teardown (zharfai.com),
section "Why video attention becomes the bottleneck".

Recipe (numpy ``Generator(Philox(seed))``, seed = 20261202 + 100*id + b for
batch element b; draw order phases, Q noise, K noise, V, g_coarse, g_fine;
all normals drawn as float32, every tensor rounded to bf16 with
round-to-nearest-even):

* iid workloads: Q, K, V ~ N(0, 1).
* field workloads: Q = 0.5*N(0,1) + sin(0.3t + 0.2x + 0.1y + phi[h, d]) and
  K likewise with the SAME phases phi[h, d] ~ U(0, 2*pi) (one phase per head
  and channel); V ~ N(0, 1).
* gates g_coarse, g_fine ~ U(0, 1), one per token and head, [B, N, H].

bf16 tensors are returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Tuple

import numpy as np

SEED_BASE = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # workload id, enters the seed
    batch: int
    heads: int
    head_dim: int
    grid: Tuple[int, int, int]   # (T, X, Y) tokens
    topk: int
    field: bool              # structured Q/K (True) or iid N(0,1) (False)
    data_wid: int = 0        # workload id whose seed the data uses (0 = own)

    @property
    def tokens(self) -> int:
        t, x, y = self.grid
        return t * x * y

    def seed(self, b: int) -> int:
        return SEED_BASE + 100 * (self.data_wid or self.wid) + b


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny_8x8x8", 1, 1, 2, 64, (8, 8, 8), 2, False),
        Workload("tiny_8x8x8_all", 1, 1, 2, 64, (8, 8, 8), 8, False, data_wid=1),
        Workload("padded_7x15x16", 2, 1, 4, 128, (7, 15, 16), 8, True),
        Workload("wan480p_dense", 3, 1, 40, 128, (21, 30, 52), 624, True),
        Workload("wan480p_vsa_k32", 4, 1, 40, 128, (21, 30, 52), 32, True, data_wid=3),
        Workload("wan720p_cfg_k64", 5, 2, 40, 128, (21, 45, 80), 64, True),
    )
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _token_coords(grid: Tuple[int, int, int]) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    t, x, y = grid
    n = np.arange(t * x * y, dtype=np.int64)
    return n // (x * y), (n // y) % x, n % y


def make_batch_element(w: Workload, b: int, heads: slice | None = None) -> Dict[str, np.ndarray]:
    """Draw one batch element: q, k, v as uint16 [N, H, D]; g_coarse, g_fine as uint16 [N, H]."""
    rng = np.random.Generator(np.random.Philox(w.seed(b)))
    n, h, d = w.tokens, w.heads, w.head_dim
    if w.field:
        phi = rng.uniform(0.0, 2.0 * math.pi, size=(h, d)).astype(np.float32)
    qn = rng.standard_normal((n, h, d), dtype=np.float32)
    kn = rng.standard_normal((n, h, d), dtype=np.float32)
    v = rng.standard_normal((n, h, d), dtype=np.float32)
    gc = rng.uniform(0.0, 1.0, size=(n, h)).astype(np.float32)
    gf = rng.uniform(0.0, 1.0, size=(n, h)).astype(np.float32)
    if w.field:
        tt, xx, yy = _token_coords(w.grid)
        base = (0.3 * tt + 0.2 * xx + 0.1 * yy).astype(np.float32)
        field = np.sin(base[:, None, None] + phi[None, :, :])
        q = np.float32(0.5) * qn + field
        k = np.float32(0.5) * kn + field
        del field
    else:
        q, k = qn, kn
    out = {
        "q": f32_to_bf16_bits(q),
        "k": f32_to_bf16_bits(k),
        "v": f32_to_bf16_bits(v),
        "g_coarse": f32_to_bf16_bits(gc),
        "g_fine": f32_to_bf16_bits(gf),
    }
    if heads is not None:
        out = {key: np.ascontiguousarray(a[:, heads]) for key, a in out.items()}
    return out


def make_inputs(w: Workload, heads: slice | None = None) -> Dict[str, np.ndarray]:
    """All batch elements stacked: q, k, v uint16 [B, N, H, D]; gates uint16 [B, N, H]."""
    parts = [make_batch_element(w, b, heads) for b in range(w.batch)]
    return {key: np.stack([p[key] for p in parts]) for key in parts[0]}


def custom_workload(name: str, batch: int, heads: int, head_dim: int,
                    grid: Tuple[int, int, int], topk: int, field: bool = True,
                    wid: int = 90) -> Workload:
    """A workload outside the named set (edge-case shapes for tests)."""
    return Workload(name, wid, batch, heads, head_dim, tuple(grid), topk, field)
