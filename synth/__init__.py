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

Recipe.  Batch element b of workload id W uses the numpy SeedSequence
20261202 + 100*W + b, spawned into six children for phases, Q noise, K
noise, V, g_coarse and g_fine; each of Q noise, K noise and V is spawned once
more into one child per head, and every child drives its own
``Generator(Philox(child))`` (so heads can be drawn in parallel).  Normals
are drawn as float32; every tensor is rounded to bf16 with
round-to-nearest-even.

* iid workloads: Q, K, V ~ N(0, 1).
* field workloads: Q = 0.5*N(0,1) + sin(0.3t + 0.2x + 0.1y + phi[h, d]) and
  K likewise with the SAME phases phi[h, d] ~ U(0, 2*pi) (one phase per head
  and channel); V ~ N(0, 1).  The field is evaluated in float32 as
  sin(a)cos(phi) + cos(a)sin(phi) with sin(a), cos(a), cos(phi), sin(phi)
  taken from float64 and rounded to float32.
* gates g_coarse, g_fine ~ U(0, 1), one per token and head, [B, N, H].

bf16 tensors are returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import math
import os
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


def _rng(seq: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(seq))


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def make_batch_element(w: Workload, b: int, heads: slice | None = None) -> Dict[str, np.ndarray]:
    """Draw one batch element: q, k, v as uint16 [N, H, D]; g_coarse, g_fine as uint16 [N, H]."""
    import torch

    n, h, d = w.tokens, w.heads, w.head_dim
    s_phi, s_q, s_k, s_v, s_gc, s_gf = np.random.SeedSequence(w.seed(b)).spawn(6)
    phi = _rng(s_phi).uniform(0.0, 2.0 * math.pi, size=(h, d)).astype(np.float32) if w.field else None
    per_head = {name: seq.spawn(h) for name, seq in (("q", s_q), ("k", s_k), ("v", s_v))}
    hsel = list(range(h) if heads is None else range(h)[heads])
    noise = {name: np.empty((len(hsel), n, d), dtype=np.float32) for name in ("q", "k", "v")}

    def draw(job):
        name, j, hh = job
        _rng(per_head[name][hh]).standard_normal(out=noise[name][j], dtype=np.float32)

    jobs = [(name, j, hh) for name in ("q", "k", "v") for j, hh in enumerate(hsel)]
    with cf.ThreadPoolExecutor(max_workers=_workers()) as ex:
        list(ex.map(draw, jobs))
    out = {}
    if w.field:
        # sin(a + phi) = sin(a) cos(phi) + cos(a) sin(phi), a = 0.3t + 0.2x + 0.1y, in float32
        tt, xx, yy = _token_coords(w.grid)
        a = 0.3 * tt + 0.2 * xx + 0.1 * yy
        sa = torch.from_numpy(np.sin(a).astype(np.float32))[None, :, None]
        ca = torch.from_numpy(np.cos(a).astype(np.float32))[None, :, None]
        ph = phi[hsel].astype(np.float64)
        cphi = torch.from_numpy(np.cos(ph).astype(np.float32))[:, None, :]
        sphi = torch.from_numpy(np.sin(ph).astype(np.float32))[:, None, :]
        field = torch.empty((len(hsel), n, d), dtype=torch.float32)
        torch.mul(sa, cphi, out=field)
        field.addcmul_(ca, sphi)
    for name in ("q", "k", "v"):
        x = torch.from_numpy(noise[name])
        if w.field and name != "v":
            x.mul_(0.5).add_(field)
        o = torch.empty((n, len(hsel), d), dtype=torch.bfloat16)
        o.copy_(x.permute(1, 0, 2))                     # round to nearest even, token-major layout
        out[name] = o.view(torch.int16).numpy().view(np.uint16)
    del noise
    gc = _rng(s_gc).uniform(0.0, 1.0, size=(n, h)).astype(np.float32)
    gf = _rng(s_gf).uniform(0.0, 1.0, size=(n, h)).astype(np.float32)
    out["g_coarse"] = np.ascontiguousarray(f32_to_bf16_bits(gc)[:, hsel])
    out["g_fine"] = np.ascontiguousarray(f32_to_bf16_bits(gf)[:, hsel])
    return out


def bf16_bits_torch(x) -> np.ndarray:
    """torch's float32 -> bf16 conversion (round to nearest, ties to even), contiguous, as bits."""
    import torch
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def make_inputs(w: Workload, heads: slice | None = None) -> Dict[str, np.ndarray]:
    """All batch elements stacked: q, k, v uint16 [B, N, H, D]; gates uint16 [B, N, H]."""
    parts = [make_batch_element(w, b, heads) for b in range(w.batch)]
    return {key: np.stack([p[key] for p in parts]) for key in parts[0]}


def custom_workload(name: str, batch: int, heads: int, head_dim: int,
                    grid: Tuple[int, int, int], topk: int, field: bool = True,
                    wid: int = 90) -> Workload:
    """A workload outside the named set (edge-case shapes for tests)."""
    return Workload(name, wid, batch, heads, head_dim, tuple(grid), topk, field)


def make_projection_inputs(w: Workload, n_tokens: int | None = None, token_offset: int = 0) -> Dict[str, np.ndarray]:
    """Raw (pre-normalisation) Q and K projections and RMSNorm weights for the pre-attention pass.

    q_raw, k_raw: uint16 [B, n_tokens, H, D], the rows of global tokens token_offset .. +n_tokens-1
    (rows past the grid, i.e. shard padding, are drawn like any other); w_q, w_k: uint16 [H*D].
    Recipe: SeedSequence SEED_BASE + 100*wid + 50 + b spawns four children per batch element (Q row
    scales, Q rows, K row scales, K rows); row r's scale is the r-th draw exp(0.7*N(0,1)) of its
    scale stream and its H*D values the r-th block of its row stream, all float32, so a shard's rows
    equal the same rows of the whole sequence; a row is its normals times its scale.  The weights
    come from SeedSequence SEED_BASE + 100*wid + 49 as 1 + 0.25*N(0,1), Q's H*D values then K's.
    All rounded to bf16 (RNE).  Meant for small and medium shapes (the draw is single-threaded)."""
    n = w.tokens - token_offset if n_tokens is None else n_tokens
    h, d = w.heads, w.head_dim
    end = token_offset + n
    out = {"q_raw": np.empty((w.batch, n, h, d), np.uint16), "k_raw": np.empty((w.batch, n, h, d), np.uint16)}
    for b in range(w.batch):
        kids = np.random.SeedSequence(SEED_BASE + 100 * (w.data_wid or w.wid) + 50 + b).spawn(4)
        for key, s_scale, s_rows in (("q_raw", kids[0], kids[1]), ("k_raw", kids[2], kids[3])):
            scale = np.exp(0.7 * _rng(s_scale).standard_normal(end, dtype=np.float32))[token_offset:]
            x = _rng(s_rows).standard_normal((end, h * d), dtype=np.float32)[token_offset:]
            out[key][b] = f32_to_bf16_bits(x * scale[:, None]).reshape(n, h, d)
    s_w = np.random.SeedSequence(SEED_BASE + 100 * (w.data_wid or w.wid) + 49)
    ww = 1.0 + 0.25 * _rng(s_w).standard_normal(2 * h * d, dtype=np.float32)
    out["w_q"] = f32_to_bf16_bits(ww[:h * d])
    out["w_k"] = f32_to_bf16_bits(ww[h * d:])
    return out
