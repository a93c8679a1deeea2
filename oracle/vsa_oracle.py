"""Plain fp64 CPU oracle for cube-based Video Sparse Attention (VSA) and dense attention.

TEST INFRASTRUCTURE ONLY.  The parity tests, the package's smoke check and
the benchmark's CPU-baseline leg call this module to obtain expected values.
The product path (the CUDA library and its Python binding) never imports,
links or runs anything here, and this module imports nothing from it.

Sources.  The method is stated in prose on the Wan2.2 real-time inference
teardown (zharfai.com, "Anatomy of the 53.6x Wan2.2 speed-up"):

* section "Why video attention becomes the bottleneck": the 480p latent grid
  is 21 frames x 30 x 52 patches = 32,760 tokens, 40 heads of width 128;
* section "Video sparse attention selects cubes": the grid is cut into
  4x4x4 cubes of 64 tokens, padded from 21x30x52 to 24x32x52 = 39,936 tokens,
  ceil(21/4)*ceil(30/4)*ceil(52/4) = 624 cubes; VSA has three parts:
  (1) coarse attention over the mean of each cube's vectors, which ranks
  candidate cubes, (2) fine token-level attention of each query cube over
  only its top-ranked key/value cubes, (3) a gated merge that keeps the fine
  result and adds a learned share of the coarse branch;
* section "Fixed-max softmax is a numerical contract": the online softmax
  keeps a running row maximum; subtracting any common constant leaves the
  probabilities unchanged.

Dense attention is softmax(q k^T / sqrt(d)) v with no causal mask (Wan2.1
acceleration article, bafh001.com, section 4.2).

Every step below is written as its definition: each function does exactly
the arithmetic of its step in float64, with numpy's matmul / sort / exp as
the only library primitives.  Readings where the pages leave a step open:

* token order n = (t*X + x)*Y + y (frame-major flattening of a (T, X, Y)
  latent grid); cubes in row-major (cube_t, cube_x, cube_y) order; tokens in
  a cube in row-major (t%4, x%4, y%4) order; padding at the high end of each
  axis;
* pooling averages the VALID tokens of a cube only (every cube holds at
  least one: padding per axis is below 4); V is pooled like Q and K so that
  the coarse branch has an output;
* the coarse scores use the same scale 1/sqrt(d) as the fine stage; cubes are
  ranked by the coarse logits; ties go to the lower cube index; the selected
  indices are returned in ascending order; the query cube's own cube is not
  forced into its selection;
* the fine softmax runs over the valid key tokens of the selected cubes
  (padded keys are excluded); a selected cube listed twice counts twice;
* the merge is O = g_coarse * O_coarse[cube] + g_fine * O_fine with one
  gate value per token and head (g_coarse = 0, g_fine = 1 when absent);
  outputs at padded positions are not defined by the method and are set to 0.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

CUBE = 4                 # cube edge in tokens
CUBE_TOKENS = CUBE ** 3  # 64 tokens per cube


# --------------------------------------------------------------------------
# bf16 input decoding (exact)
# --------------------------------------------------------------------------
def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    u32 = np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Step a1: grid, cubes, padding, tiling  ("Video sparse attention selects cubes")
# --------------------------------------------------------------------------
def padded_grid(grid: Tuple[int, int, int]) -> Tuple[int, int, int]:
    """Each axis rounded up to a multiple of the cube edge (21x30x52 -> 24x32x52)."""
    return tuple(CUBE * math.ceil(a / CUBE) for a in grid)


def cube_grid(grid: Tuple[int, int, int]) -> Tuple[int, int, int]:
    """Cubes per axis: (ceil(T/4), ceil(X/4), ceil(Y/4)) (6x8x13 at 480p)."""
    return tuple(math.ceil(a / CUBE) for a in grid)


def num_cubes(grid: Tuple[int, int, int]) -> int:
    ct, cx, cy = cube_grid(grid)
    return ct * cx * cy


def padded_tokens(grid: Tuple[int, int, int]) -> int:
    return num_cubes(grid) * CUBE_TOKENS


def tile_source_index(grid: Tuple[int, int, int]) -> np.ndarray:
    """For every cube-major position p = c*64 + o, the source token n, or -1 for padding.

    c = ((t//4)*Xc + x//4)*Yc + y//4 and o = ((t%4)*4 + x%4)*4 + y%4.
    """
    T, X, Y = grid
    _, Xc, Yc = cube_grid(grid)
    p = np.arange(padded_tokens(grid), dtype=np.int64)
    c, o = p // CUBE_TOKENS, p % CUBE_TOKENS
    c_t, c_x, c_y = c // (Xc * Yc), (c // Yc) % Xc, c % Yc
    o_t, o_x, o_y = o // 16, (o // 4) % 4, o % 4
    t, x, y = CUBE * c_t + o_t, CUBE * c_x + o_x, CUBE * c_y + o_y
    valid = (t < T) & (x < X) & (y < Y)
    n = (t * X + x) * Y + y
    return np.where(valid, n, -1)


def tile(x: np.ndarray, grid: Tuple[int, int, int]) -> np.ndarray:
    """[B, N, H, D] -> cube-major [B, H, Npad, D]; padded rows are zero."""
    src = tile_source_index(grid)
    B, N, H, D = x.shape
    out = np.zeros((B, H, src.size, D), dtype=x.dtype)
    valid = src >= 0
    out[:, :, valid, :] = np.transpose(x[:, src[valid], :, :], (0, 2, 1, 3))
    return out


def untile(xt: np.ndarray, grid: Tuple[int, int, int]) -> np.ndarray:
    """Inverse of tile on the valid positions: [B, H, Npad, D] -> [B, N, H, D]."""
    src = tile_source_index(grid)
    valid = src >= 0
    B, H, _, D = xt.shape
    N = int(np.prod(grid))
    out = np.empty((B, N, H, D), dtype=xt.dtype)
    out[:, src[valid], :, :] = np.transpose(xt[:, :, valid, :], (0, 2, 1, 3))
    return out


def key_valid_mask(grid: Tuple[int, int, int]) -> np.ndarray:
    """[Npad] bool: True where the cube-major position holds a real token."""
    return tile_source_index(grid) >= 0


def valid_counts(grid: Tuple[int, int, int]) -> np.ndarray:
    """[C] number of real tokens in each cube (1..64)."""
    return key_valid_mask(grid).reshape(-1, CUBE_TOKENS).sum(axis=1)


# --------------------------------------------------------------------------
# Step a2: cube mean-pooling  (coarse part (1): one representative per cube)
# --------------------------------------------------------------------------
def pool(xt: np.ndarray, grid: Tuple[int, int, int]) -> np.ndarray:
    """[B, H, Npad, D] -> [B, H, C, D]: mean over the valid tokens of each cube."""
    B, H, Npad, D = xt.shape
    mask = key_valid_mask(grid).reshape(-1, CUBE_TOKENS)             # [C, 64]
    cubes = xt.reshape(B, H, -1, CUBE_TOKENS, D)
    sums = np.einsum("bhcod,co->bhcd", cubes, mask.astype(xt.dtype))
    return sums / mask.sum(axis=1)[None, None, :, None]


# --------------------------------------------------------------------------
# Step a3: coarse cube attention  (coarse part (1): cheap block-level attention)
# --------------------------------------------------------------------------
def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted (exact algebra, no overflow)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def coarse(qbar: np.ndarray, kbar: np.ndarray, vbar: np.ndarray, scale: float):
    """S_c = scale * Qbar Kbar^T  [B,H,C,C];  O_c = softmax_rows(S_c) Vbar  [B,H,C,D]."""
    scores = scale * np.matmul(qbar, np.swapaxes(kbar, -1, -2))
    o_coarse = np.matmul(softmax_rows(scores), vbar)
    return scores, o_coarse


# --------------------------------------------------------------------------
# Step a4: top-k cube selection  (rank candidates, keep the k highest)
# --------------------------------------------------------------------------
def topk(scores: np.ndarray, k: int) -> np.ndarray:
    """[..., C] scores -> int32 [..., k]: the k largest entries per row.

    Equal scores are ranked by the lower cube index (a stable sort of the
    negated scores keeps index order among equals); the kept indices are
    returned in ascending order.
    """
    order = np.argsort(-scores, axis=-1, kind="stable")[..., :k]
    return np.sort(order, axis=-1).astype(np.int32)


def kth_gap(scores: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per row: the k-th and (k+1)-th largest score (for the near-tie rule)."""
    s = -np.sort(-scores, axis=-1)
    kth = s[..., k - 1]
    nxt = s[..., k] if k < scores.shape[-1] else np.full(kth.shape, -np.inf)
    return kth, nxt


# --------------------------------------------------------------------------
# Step a5 / a8: fine attention over the selected cubes  (fine part (2))
# --------------------------------------------------------------------------
def fine_cube(q_cube: np.ndarray, k_head: np.ndarray, v_head: np.ndarray,
              selected: Sequence[int], key_valid: np.ndarray, scale: float):
    """One query cube against the tokens of its selected key cubes.

    q_cube [64, D]; k_head, v_head [Npad, D] (cube-major); key_valid [Npad].
    Returns (O [64, D], lse [64]) with lse = log(sum_j exp(scale * q . k_j))
    over the valid keys j of the selected cubes.
    """
    rows = np.concatenate([np.arange(c * CUBE_TOKENS, (c + 1) * CUBE_TOKENS) for c in selected])
    rows = rows[key_valid[rows]]
    s = scale * (q_cube @ k_head[rows].T)                       # [64, nkeys]
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    denom = np.sum(e, axis=-1, keepdims=True)
    o = (e / denom) @ v_head[rows]
    lse = m[:, 0] + np.log(denom[:, 0])
    return o, lse


def fine(qt: np.ndarray, kt: np.ndarray, vt: np.ndarray, idx: Optional[np.ndarray],
         scale: float, grid: Tuple[int, int, int],
         items: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Fine stage on tiled tensors [B, H, Npad, D].

    idx [B, H, C, k] selected key cubes per query cube, or None for all C
    cubes (dense attention).  ``items`` restricts the work to the listed
    (b, h, query_cube) triples; other rows of the result are NaN.
    Returns (O_fine [B, H, Npad, D], lse [B, H, Npad]).  Rows of padded query
    positions are computed like any other row (their Q is zero) but carry no
    meaning.
    """
    B, H, Npad, D = qt.shape
    C = Npad // CUBE_TOKENS
    kv = key_valid_mask(grid)
    o = np.full(qt.shape, np.nan)
    lse = np.full((B, H, Npad), np.nan)
    if items is None:
        items = [(b, h, i) for b in range(B) for h in range(H) for i in range(C)]
    for b, h, i in items:
        sel = range(C) if idx is None else idx[b, h, i]
        r = slice(i * CUBE_TOKENS, (i + 1) * CUBE_TOKENS)
        o[b, h, r], lse[b, h, r] = fine_cube(qt[b, h, r], kt[b, h], vt[b, h], sel, kv, scale)
    return o, lse


# --------------------------------------------------------------------------
# Step a6: gated merge  (part (3))
# --------------------------------------------------------------------------
def combine(o_coarse: np.ndarray, o_fine: np.ndarray, g_coarse: Optional[np.ndarray],
            g_fine: Optional[np.ndarray], grid: Tuple[int, int, int]) -> np.ndarray:
    """O[p] = g_coarse[n(p)] * O_coarse[cube(p)] + g_fine[n(p)] * O_fine[p], per head.

    o_coarse [B,H,C,D], o_fine [B,H,Npad,D], gates [B,N,H] (token order) or
    None.  Padded positions are set to zero.
    """
    B, H, Npad, D = o_fine.shape
    src = tile_source_index(grid)
    valid = src >= 0
    oc = np.repeat(o_coarse, CUBE_TOKENS, axis=2)               # [B,H,Npad,D]
    gc = np.zeros((B, H, Npad))
    gf = np.ones((B, H, Npad))
    if g_coarse is not None:
        gc[:, :, valid] = np.transpose(g_coarse[:, src[valid], :], (0, 2, 1))
    if g_fine is not None:
        gf[:, :, valid] = np.transpose(g_fine[:, src[valid], :], (0, 2, 1))
    out = gc[..., None] * oc + gf[..., None] * o_fine
    out[:, :, ~valid, :] = 0.0
    return out


# --------------------------------------------------------------------------
# Whole call (a1 .. a7) and dense attention (a8)
# --------------------------------------------------------------------------
def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Tuple[int, int, int],
            topk_k: int, scale: Optional[float] = None,
            g_coarse: Optional[np.ndarray] = None, g_fine: Optional[np.ndarray] = None,
            idx_override: Optional[np.ndarray] = None):
    """VSA on float64 inputs q, k, v [B, N, H, D]; gates [B, N, H] or None.

    Returns a dict with every intermediate: qt, kt, vt, qbar, kbar, vbar,
    scores, o_coarse, idx, o_fine, lse, o_tiled, out [B, N, H, D].
    ``idx_override`` replaces the computed selection in the fine stage (used
    to compare outputs when a near-tie legitimately swapped a cube).
    """
    D = q.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    r = {"qt": tile(q, grid), "kt": tile(k, grid), "vt": tile(v, grid)}
    r["qbar"], r["kbar"], r["vbar"] = (pool(r[n], grid) for n in ("qt", "kt", "vt"))
    r["scores"], r["o_coarse"] = coarse(r["qbar"], r["kbar"], r["vbar"], scale)
    r["idx"] = topk(r["scores"], topk_k)
    use = r["idx"] if idx_override is None else idx_override
    r["o_fine"], r["lse"] = fine(r["qt"], r["kt"], r["vt"], use, scale, grid)
    r["o_tiled"] = combine(r["o_coarse"], r["o_fine"], g_coarse, g_fine, grid)
    r["out"] = untile(r["o_tiled"], grid)
    return r


def dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Tuple[int, int, int],
          scale: Optional[float] = None):
    """Dense bidirectional attention through the cube path: every cube selected, no gates.

    Returns (out [B, N, H, D], lse [B, N, H]).
    """
    D = q.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qt, kt, vt = tile(q, grid), tile(k, grid), tile(v, grid)
    o, lse = fine(qt, kt, vt, None, scale, grid)
    out = untile(o, grid)
    lse_t = untile(lse[..., None], grid)[..., 0]
    return out, lse_t
