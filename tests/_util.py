"""Helpers shared by the GPU parity tests: host<->device bf16 moves and the tolerance checks."""
import dataclasses
import math

import numpy as np
import torch

from oracle import vsa_oracle as O

# Output tolerances for bf16 results against the fp64 oracle (per head, over
# real tokens): max |err| <= 2e-2 and ||err|| / ||ref|| <= 5e-3; log-sum-exp
# |err| <= 1e-3; float32 coarse output relative L2 <= 1e-5.
MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3
COARSE_REL_L2 = 1e-5
NEAR_TIE_REL = 1e-5
# share of a comparison's rows that may differ from the oracle's selection through near-ties
MAX_EXCUSED_SHARE = 0.02


def to_dev(u16: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_dev(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> float64 numpy (bf16 decoded exactly)."""
    if t.dtype == torch.bfloat16:
        return O.bf16_to_f64(bf16_bits(t))
    return t.detach().cpu().numpy().astype(np.float64)


def check_close(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, rel_l2=REL_L2):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    ma = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rl = float(np.linalg.norm(got - ref)) / denom if denom > 0 else float(np.linalg.norm(got - ref))
    assert ma <= max_abs, f"{what}: max abs err {ma:.3e} > {max_abs}"
    assert rl <= rel_l2, f"{what}: rel L2 err {rl:.3e} > {rel_l2}"
    return ma, rl


def check_heads(got_tiled: np.ndarray, ref_tiled: np.ndarray, grid, what: str):
    """Per (b, h) tolerance check over the real (unpadded) rows of tiled [B,H,Npad,D] arrays."""
    valid = O.key_valid_mask(grid)
    worst = (0.0, 0.0)
    for b in range(got_tiled.shape[0]):
        for h in range(got_tiled.shape[1]):
            ma, rl = check_close(got_tiled[b, h, valid], ref_tiled[b, h, valid], f"{what}[b={b},h={h}]")
            worst = (max(worst[0], ma), max(worst[1], rl))
    return worst


@dataclasses.dataclass
class NearTie:
    """Outcome of comparing a GPU selection with the oracle's under the near-tie rule."""
    ok: np.ndarray      # bool per row: identical, or different only through a documented near-tie
    rows: int           # rows compared
    differ: int         # rows whose selections differ
    excused: int        # rows that differ and that the near-tie rule accepts


# every comparison of the session: (label, rows, rows excused as near-ties, rows that failed);
# tests/conftest.py prints it in the terminal summary
NEAR_TIE_LOG = []


def near_tie_check(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, k: int,
                   label: str = "") -> NearTie:
    """Rows where the GPU selection differs from the oracle's only through a documented near-tie.

    A row may differ only if the oracle's k-th and (k+1)-th scores are within
    1e-5 relative, and only in cubes whose oracle scores lie within that band
    of the k-th score.  The counts are appended to NEAR_TIE_LOG.
    """
    kth, nxt = O.kth_gap(ora_scores, k)
    band = NEAR_TIE_REL * np.maximum(np.abs(kth), np.abs(nxt))
    ok = np.ones(gpu_idx.shape[:-1], dtype=bool)
    differ = 0
    for pos in np.ndindex(*gpu_idx.shape[:-1]):
        g, o = set(gpu_idx[pos].tolist()), set(ora_idx[pos].tolist())
        if g == o:
            continue
        differ += 1
        if not (abs(kth[pos] - nxt[pos]) < band[pos]):
            ok[pos] = False
            continue
        row = ora_scores[pos]
        for c in g.symmetric_difference(o):
            if abs(row[c] - kth[pos]) > band[pos]:
                ok[pos] = False
    failed = int((~ok).sum())
    r = NearTie(ok=ok, rows=int(ok.size), differ=differ, excused=differ - failed)
    NEAR_TIE_LOG.append((label, r.rows, r.excused, failed))
    return r


def assert_selection(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, k: int,
                     label: str) -> NearTie:
    """Every row identical or a documented near-tie, and at most MAX_EXCUSED_SHARE of the rows excused."""
    r = near_tie_check(gpu_idx, ora_idx, ora_scores, k, label)
    assert r.ok.all(), f"{label}: {r.rows - int(r.ok.sum())} of {r.rows} rows differ beyond the near-tie rule"
    assert r.excused <= MAX_EXCUSED_SHARE * r.rows, \
        f"{label}: {r.excused} of {r.rows} rows excused as near-ties (more than {MAX_EXCUSED_SHARE:.0%})"
    return r


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
