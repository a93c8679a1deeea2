"""Pins for the fp64 oracle, checked against things other than the oracle itself.

* values printed on the Wan2.2 teardown page (tests/golden/page_facts.txt);
* hand-worked index maps and pooled values;
* library routines the method reduces to: torch's scaled_dot_product_attention
  (dense attention, coarse attention on pooled vectors) and torch's logsumexp;
* closed forms (zero queries, constant values, duplicated selections);
* brute force on tiny inputs (top-k by Python tuple sorting);
* a few planted mistakes in the oracle that these pins must catch.
"""
import math
import os

import numpy as np
import pytest
import torch

import synth
from oracle import vsa_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _f64(w, heads=None):
    x = synth.make_inputs(w, heads)
    return {k: O.bf16_to_f64(v) for k, v in x.items()}


def _sdpa(q, k, v, scale=None):
    """torch's fp64 CPU scaled-dot-product attention on [B, N, H, D] arrays."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(np.transpose(a, (0, 2, 1, 3)))) for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    return np.transpose(o.numpy(), (0, 2, 1, 3))


# ---------------------------------------------------------------- page facts
def _facts():
    out = {}
    with open(os.path.join(HERE, "golden", "page_facts.txt")) as f:
        for line in f:
            line = line.split("|")[0].strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("="))
            out[key] = val
    return out


def test_page_facts_480p_grid():
    f = _facts()
    grid = (21, 30, 52)
    assert (81 - 1) // 4 + 1 == int(f["latent_frames_from_81"])
    assert int(np.prod(grid)) == int(f["tokens_480p"])
    assert "x".join(map(str, O.padded_grid(grid))) == f["padded_grid_480p"]
    assert O.padded_tokens(grid) == int(f["padded_tokens_480p"])
    assert "x".join(map(str, O.cube_grid(grid))) == f["cube_grid_480p"]
    assert O.num_cubes(grid) == int(f["cubes_480p"])
    assert O.CUBE_TOKENS == int(f["tokens_per_cube"])
    assert round(O.num_cubes(grid) * (1 - 0.875)) == int(f["selected_at_87_5_percent"])
    assert O.num_cubes(grid) * int(f["heads_480p"]) == int(f["output_tiles_480p"])
    assert round(int(f["tokens_480p"]) ** 2 / 1e9, 2) == float(f["scores_per_head_billion"])
    # the tile map covers every token once and pads the rest
    src = O.tile_source_index(grid)
    assert src.size == 39936 and (src >= 0).sum() == 32760
    assert np.array_equal(np.sort(src[src >= 0]), np.arange(32760))


def test_page_facts_roofline_numbers():
    f = _facts()
    grid, heads, d, k = (21, 30, 52), 40, 128, 78
    n_valid = int(np.prod(grid))
    # QK^T and PV: 2 matmuls x 2 flop per multiply-add, over the valid query tokens
    flops = 4 * d * heads * n_valid * k * O.CUBE_TOKENS
    assert abs(flops / 1e12 - float(f["tflop_at_78_cubes"])) < 0.01
    # K and V cube tiles streamed once per (query cube, head, selected cube)
    kv_bytes = O.num_cubes(grid) * heads * k * O.CUBE_TOKENS * d * 2 * 2
    assert abs(kv_bytes / 1e9 - float(f["kv_stream_gb_at_78_cubes"])) < 0.5


# ---------------------------------------------------------------- tile map
@pytest.mark.parametrize("grid,token,expect_p", [
    ((8, 8, 8), (0, 0, 4), 64),                    # cube (0,0,1) = cube 1, offset 0
    ((8, 8, 8), (1, 2, 3), 27),                    # cube 0, offset (1*4+2)*4+3
    ((8, 8, 8), (5, 6, 7), 7 * 64 + 27),           # cube (1,1,1) = 7
    ((7, 15, 16), (6, 14, 15), 31 * 64 + 43),      # last token of the padded-small grid
    ((7, 15, 16), (0, 4, 0), 4 * 64 + 0),          # cube (0,1,0) = 4
    ((21, 30, 52), (20, 29, 51), 623 * 64 + 0 * 16 + 1 * 4 + 3),
])
def test_tile_map_hand_examples(grid, token, expect_p):
    t, x, y = token
    n = (t * grid[1] + x) * grid[2] + y
    src = O.tile_source_index(grid)
    assert src[expect_p] == n
    assert np.count_nonzero(src == n) == 1


def test_tile_map_padding_positions():
    src = O.tile_source_index((7, 15, 16))
    assert src[31 * 64 + 63] == -1                 # (t,x,y) = (7,15,15): t and x padded
    assert src[1 * 64 + 0] == 4                    # cube (0,0,1) offset 0 -> token (0,0,4)
    assert (src >= 0).sum() == 7 * 15 * 16


def test_untile_tile_roundtrip_and_zero_padding():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)["q"]
    xt = O.tile(x, w.grid)
    assert np.array_equal(O.untile(xt, w.grid), x)
    assert np.all(xt[:, :, ~O.key_valid_mask(w.grid), :] == 0)


@pytest.mark.parametrize("grid,expected", [
    ((7, 15, 16), {64, 48, 36}),
    ((21, 30, 52), {64, 32, 16, 8}),
    ((21, 45, 80), {64, 16, 4}),
    ((8, 8, 8), {64}),
])
def test_valid_counts(grid, expected):
    vc = O.valid_counts(grid)
    assert set(vc.tolist()) == expected
    assert vc.sum() == int(np.prod(grid)) and vc.min() >= 1


# ---------------------------------------------------------------- pooling
def test_pool_partial_cube_hand_value():
    # grid 5x4x4: cube 1 holds one valid frame (t=4) of 16 tokens
    grid = (5, 4, 4)
    N = 80
    x = np.zeros((1, N, 1, 2))
    x[0, :, 0, 0] = np.arange(N)            # channel 0 = token index
    x[0, :, 0, 1] = 1.0                     # channel 1 = constant
    xbar = O.pool(O.tile(x, grid), grid)
    assert xbar.shape == (1, 1, 2, 2)
    assert xbar[0, 0, 0, 0] == pytest.approx(np.mean(np.arange(64)))
    assert xbar[0, 0, 1, 0] == pytest.approx(np.mean(np.arange(64, 80)))   # valid tokens only
    assert np.all(xbar[0, 0, :, 1] == 1.0)


# ---------------------------------------------------------------- coarse
def test_coarse_equals_library_attention_on_pooled_vectors():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    qb, kb, vb = (O.pool(O.tile(x[n], w.grid), w.grid) for n in ("q", "k", "v"))
    scale = 1 / math.sqrt(w.head_dim)
    scores, oc = O.coarse(qb, kb, vb, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qb), torch.from_numpy(kb), torch.from_numpy(vb)).numpy()
    np.testing.assert_allclose(oc, ref, rtol=1e-12, atol=1e-12)
    # score (i, j) is query cube i against key cube j
    i, j = 3, 17
    assert scores[0, 1, i, j] == pytest.approx(scale * np.dot(qb[0, 1, i], kb[0, 1, j]), rel=1e-13)


def test_coarse_rows_sum_to_one_and_zero_query():
    rng = np.random.default_rng(0)
    qb = np.zeros((1, 1, 6, 8))
    kb, vb = rng.normal(size=(1, 1, 6, 8)), rng.normal(size=(1, 1, 6, 8))
    s, oc = O.coarse(qb, kb, vb, 0.5)
    assert np.all(s == 0)
    np.testing.assert_allclose(oc[0, 0], np.tile(vb[0, 0].mean(axis=0), (6, 1)), rtol=1e-13)
    p = O.softmax_rows(rng.normal(size=(5, 7)) * 30)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- top-k
@pytest.mark.parametrize("row,k,expect", [
    ([3.0, 1.0, 3.0, 2.0, 3.0], 2, [0, 2]),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 3, [0, 2, 4]),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 4, [0, 2, 3, 4]),
    ([0.0, 0.0, 0.0, 0.0], 2, [0, 1]),
    ([-1.0, -5.0, -0.5, -2.0], 1, [2]),
    ([1.0, 2.0, 3.0, 4.0], 4, [0, 1, 2, 3]),
    ([-0.0, 0.0, -0.0], 1, [0]),
])
def test_topk_hand_examples(row, k, expect):
    assert O.topk(np.array(row), k).tolist() == expect


def test_topk_brute_force_tuples():
    rng = np.random.default_rng(1)
    for _ in range(200):
        C = int(rng.integers(1, 12))
        k = int(rng.integers(1, C + 1))
        row = rng.integers(-3, 4, size=C).astype(float)     # many ties
        ranked = sorted(range(C), key=lambda j: (-row[j], j))
        assert O.topk(row, k).tolist() == sorted(ranked[:k])


def test_kth_value_is_the_smallest_selected_and_next_the_largest_left_out():
    """kth_gap agrees with topk's own selection: the k-th largest score is the
    smallest selected one and the (k+1)-th the largest left out (-inf at k = C)."""
    rng = np.random.default_rng(5)
    scores = rng.integers(-4, 5, size=(3, 2, 9)).astype(float) + rng.normal(size=(3, 2, 9)) * (rng.random((3, 2, 9)) < 0.5)
    for k in range(1, 10):
        kth, nxt = O.kth_gap(scores, k)
        sel = O.topk(scores, k)
        for pos in np.ndindex(*scores.shape[:-1]):
            row = scores[pos]
            chosen = row[sel[pos]]
            rest = np.delete(row, sel[pos])
            assert kth[pos] == chosen.min()
            assert nxt[pos] == (rest.max() if rest.size else -np.inf)


# ---------------------------------------------------------------- near-tie rule inputs
@pytest.mark.parametrize("row,k,expect", [
    ([3.0, 1.0, 3.0, 2.0, 3.0], 1, (3.0, 3.0)),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 2, (3.0, 3.0)),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 3, (3.0, 2.0)),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 4, (2.0, 1.0)),
    ([3.0, 1.0, 3.0, 2.0, 3.0], 5, (1.0, -math.inf)),    # k = C: nothing is left out
    ([0.5, -1.0, 2.0, 7.0], 1, (7.0, 2.0)),
    ([0.5, -1.0, 2.0, 7.0], 2, (2.0, 0.5)),
    ([-4.0, -2.5, -3.0], 2, (-3.0, -4.0)),
    ([1.0, 1.0 + 1e-9, 0.0], 1, (1.0 + 1e-9, 1.0)),
])
def test_kth_gap_hand_rows(row, k, expect):
    """k-th and (k+1)-th largest entries of hand rows (counted with repeats)."""
    kth, nxt = O.kth_gap(np.array(row), k)
    assert (float(kth), float(nxt)) == expect


def test_kth_gap_brute_force_tuples():
    """Random tie-heavy rows, several leading axes: Python's sorted() gives the two values."""
    rng = np.random.default_rng(2)
    for _ in range(100):
        C = int(rng.integers(1, 10))
        k = int(rng.integers(1, C + 1))
        a = rng.integers(-3, 4, size=(2, 3, C)).astype(float)
        kth, nxt = O.kth_gap(a, k)
        for pos in np.ndindex(2, 3):
            desc = sorted(a[pos].tolist(), reverse=True)
            assert kth[pos] == desc[k - 1]
            assert nxt[pos] == (desc[k] if k < C else -math.inf)


# ---------------------------------------------------------------- bf16 decoding
# bit pattern -> exact value (sign bit, 8 exponent bits with bias 127, 7 fraction bits)
BF16_TABLE = [
    (0x0000, 0.0), (0x3F80, 1.0), (0xBF80, -1.0), (0xC040, -3.0), (0x3F00, 0.5), (0x4120, 10.0),
    (0x4049, 3.140625), (0x3C00, 2.0 ** -7), (0x0080, 2.0 ** -126), (0x0001, 2.0 ** -133),
    (0x007F, 127 * 2.0 ** -133), (0x8001, -(2.0 ** -133)), (0x7F7F, (2 - 2 ** -7) * 2.0 ** 127),
    (0xFF7F, -(2 - 2 ** -7) * 2.0 ** 127), (0x7F80, math.inf), (0xFF80, -math.inf), (0x3FC0, 1.5),
    (0x4B00, 2.0 ** 23), (0x4B01, 2.0 ** 23 + 2.0 ** 16),
]


def test_bf16_decode_table():
    got = O.bf16_to_f64(np.array([b for b, _ in BF16_TABLE], dtype=np.uint16))
    assert got.dtype == np.float64
    assert got.tolist() == [v for _, v in BF16_TABLE]
    z = O.bf16_to_f64(np.array([0x0000, 0x8000], dtype=np.uint16))
    assert z.tolist() == [0.0, 0.0] and not np.signbit(z[0]) and np.signbit(z[1])
    assert np.isnan(O.bf16_to_f64(np.array([0x7FC0, 0xFFC1, 0x7F81], dtype=np.uint16))).all()


def _bf16_by_fields(u: int) -> float:
    sign = -1.0 if u >> 15 else 1.0
    e, f = (u >> 7) & 0xFF, u & 0x7F
    if e == 0xFF:
        return sign * math.inf if f == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(f, -133)                 # subnormal: f / 128 * 2^-126
    return sign * math.ldexp(128 + f, e - 134)            # (1 + f/128) * 2^(e - 127)


def test_bf16_decode_every_pattern_by_fields():
    u = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = O.bf16_to_f64(u)
    ref = np.array([_bf16_by_fields(int(b)) for b in range(1 << 16)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ---------------------------------------------------------------- fine / dense
@pytest.mark.parametrize("name", ["tiny_8x8x8", "padded_7x15x16"])
def test_dense_equals_library_sdpa(name):
    w = synth.WORKLOADS[name]
    x = _f64(w)
    out, lse = O.dense(x["q"], x["k"], x["v"], w.grid)
    np.testing.assert_allclose(out, _sdpa(x["q"], x["k"], x["v"]), rtol=1e-10, atol=1e-12)
    scale = 1 / math.sqrt(w.head_dim)
    qh, kh = (np.transpose(x[n], (0, 2, 1, 3)) for n in ("q", "k"))
    s = scale * np.matmul(qh, np.swapaxes(kh, -1, -2))
    ref_lse = np.transpose(torch.logsumexp(torch.from_numpy(s), dim=-1).numpy(), (0, 2, 1))
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny_8x8x8_all", "padded_7x15x16"])
def test_vsa_with_all_cubes_and_no_gates_is_dense(name):
    w = synth.WORKLOADS[name]
    x = _f64(w)
    C = O.num_cubes(w.grid)
    r = O.forward(x["q"], x["k"], x["v"], w.grid, C)
    assert np.array_equal(r["idx"][0, 0, 0], np.arange(C))
    np.testing.assert_allclose(r["out"], _sdpa(x["q"], x["k"], x["v"]), rtol=1e-10, atol=1e-12)


def test_fine_single_cube_against_library():
    # one query cube, two selected key cubes: equals SDPA on exactly those tokens
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    qt, kt, vt = (O.tile(x[n], w.grid) for n in ("q", "k", "v"))
    kv = O.key_valid_mask(w.grid)
    sel = [5, 31]
    rows = np.concatenate([np.arange(c * 64, c * 64 + 64) for c in sel])
    rows = rows[kv[rows]]
    o, _ = O.fine_cube(qt[0, 2, 64:128], kt[0, 2], vt[0, 2], sel, kv, 1 / math.sqrt(128))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qt[0, 2, 64:128]), torch.from_numpy(kt[0, 2, rows]),
        torch.from_numpy(vt[0, 2, rows])).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_zero_query_closed_form():
    """Q = 0: all scores 0, ties select cubes 0..k-1, O_fine = mean of their valid V."""
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    q = np.zeros_like(x["q"])
    k_sel = 5
    r = O.forward(q, x["k"], x["v"], w.grid, k_sel)
    C = O.num_cubes(w.grid)
    assert np.array_equal(r["idx"], np.broadcast_to(np.arange(k_sel), (1, w.heads, C, k_sel)))
    # tokens of cubes 0..k-1 straight from the grid coordinates
    T, X, Y = w.grid
    _, Xc, Yc = O.cube_grid(w.grid)
    members = [(t * X + xx) * Y + y for t in range(T) for xx in range(X) for y in range(Y)
               if ((t // 4) * Xc + xx // 4) * Yc + y // 4 < k_sel]
    mean_v = x["v"][0, members].mean(axis=0)                       # [H, D]
    np.testing.assert_allclose(r["out"][0], np.broadcast_to(mean_v, r["out"][0].shape), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r["lse"][:, :, O.key_valid_mask(w.grid)], math.log(len(members)), rtol=1e-13)
    vbar = r["vbar"][0]                                            # [H, C, D]
    np.testing.assert_allclose(r["o_coarse"][0], np.broadcast_to(vbar.mean(axis=1, keepdims=True), vbar.shape),
                               rtol=1e-11, atol=1e-12)


def test_constant_values_give_constant_output():
    w = synth.WORKLOADS["tiny_8x8x8"]
    x = _f64(w)
    r = O.forward(x["q"], x["k"], np.ones_like(x["v"]), w.grid, 2)
    np.testing.assert_allclose(r["out"], 1.0, rtol=1e-13)


def test_duplicated_selection_counts_twice():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    qt, kt, vt = (O.tile(x[n], w.grid) for n in ("q", "k", "v"))
    kv = O.key_valid_mask(w.grid)
    s = 1 / math.sqrt(128)
    o1, l1 = O.fine_cube(qt[0, 0, :64], kt[0, 0], vt[0, 0], [2, 9], kv, s)
    o2, l2 = O.fine_cube(qt[0, 0, :64], kt[0, 0], vt[0, 0], [2, 9, 2, 9], kv, s)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + math.log(2), rtol=1e-13)


def test_padded_keys_are_ignored():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    qt, kt, vt = (O.tile(x[n], w.grid) for n in ("q", "k", "v"))
    kv = O.key_valid_mask(w.grid)
    idx = O.topk(O.coarse(*(O.pool(t, w.grid) for t in (qt, kt, vt)), 1 / math.sqrt(128))[0], 8)
    o1, l1 = O.fine(qt, kt, vt, idx, 1 / math.sqrt(128), w.grid)
    kt2 = kt.copy()
    kt2[:, :, ~kv, :] = 1e4
    o2, l2 = O.fine(qt, kt2, vt, idx, 1 / math.sqrt(128), w.grid)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_overflow_scores_stay_finite_and_match_library():
    """Scores near 150 overflow an unshifted fp32 exp; the shifted softmax does not."""
    w = synth.WORKLOADS["tiny_8x8x8"]
    x = _f64(w)
    q, k = x["q"] * 12.0, x["k"] * 12.0
    out, lse = O.dense(q, k, x["v"], w.grid)
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    s = np.einsum("bnhd,bmhd->bhnm", q, k) / 8.0
    assert s.max() > 100
    np.testing.assert_allclose(out, _sdpa(q, k, x["v"]), rtol=1e-9, atol=1e-12)


def test_combine_hand_value():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = _f64(w)
    r = O.forward(x["q"], x["k"], x["v"], w.grid, 8, g_coarse=x["g_coarse"], g_fine=x["g_fine"])
    t, xx, y, h = 6, 13, 9, 3
    n = (t * 15 + xx) * 16 + y
    cube = ((t // 4) * 4 + xx // 4) * 4 + y // 4
    p = cube * 64 + ((t % 4) * 4 + xx % 4) * 4 + y % 4
    expect = x["g_coarse"][0, n, h] * r["o_coarse"][0, h, cube] + x["g_fine"][0, n, h] * r["o_fine"][0, h, p]
    np.testing.assert_allclose(r["out"][0, n, h], expect, rtol=1e-14)


# ---------------------------------------------------------------- planted mistakes
def _pins_pass():
    try:
        test_tile_map_hand_examples((8, 8, 8), (1, 2, 3), 27)
        test_tile_map_hand_examples((7, 15, 16), (6, 14, 15), 31 * 64 + 43)
        test_pool_partial_cube_hand_value()
        test_coarse_equals_library_attention_on_pooled_vectors()
        test_topk_hand_examples([3.0, 1.0, 3.0, 2.0, 3.0], 2, [0, 2])
        test_dense_equals_library_sdpa("padded_7x15x16")
        test_zero_query_closed_form()
        test_combine_hand_value()
        test_kth_gap_hand_rows([3.0, 1.0, 3.0, 2.0, 3.0], 3, (3.0, 2.0))
        test_kth_gap_hand_rows([3.0, 1.0, 3.0, 2.0, 3.0], 5, (1.0, -math.inf))
        test_kth_gap_hand_rows([0.5, -1.0, 2.0, 7.0], 2, (2.0, 0.5))
        test_bf16_decode_table()
    except AssertionError:
        return False
    return True


def test_pins_pass_on_the_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("mutation", ["swap_xy", "pool_all64", "transpose_coarse",
                                      "topk_smallest", "no_scale", "swap_gates", "keep_padded_keys",
                                      "kth_off_by_one", "kth_unsorted", "kth_ascending",
                                      "bf16_shift15", "bf16_no_sign"])
def test_planted_mistake_is_caught(monkeypatch, mutation):
    good = {n: getattr(O, n) for n in ("tile_source_index", "pool", "coarse", "topk", "fine_cube", "combine",
                                       "kth_gap", "bf16_to_f64")}
    if mutation == "swap_xy":
        def bad(grid):
            T, X, Y = grid
            if X == Y:
                return good["tile_source_index"](grid)
            src = good["tile_source_index"]((T, Y, X))
            return np.where(src >= 0, src, -1)
        monkeypatch.setattr(O, "tile_source_index", bad)
    elif mutation == "pool_all64":
        monkeypatch.setattr(O, "pool", lambda xt, grid: xt.reshape(*xt.shape[:2], -1, 64, xt.shape[-1]).mean(axis=3))
    elif mutation == "transpose_coarse":
        monkeypatch.setattr(O, "coarse", lambda q, k, v, s: good["coarse"](k, q, v, s))
    elif mutation == "topk_smallest":
        monkeypatch.setattr(O, "topk", lambda s, k: good["topk"](-s, k))
    elif mutation == "no_scale":
        monkeypatch.setattr(O, "fine_cube", lambda q, k, v, sel, kv, s: good["fine_cube"](q, k, v, sel, kv, 1.0))
    elif mutation == "swap_gates":
        monkeypatch.setattr(O, "combine", lambda oc, of, gc, gf, grid: good["combine"](oc, of, gf, gc, grid))
    elif mutation == "keep_padded_keys":
        monkeypatch.setattr(O, "fine_cube",
                            lambda q, k, v, sel, kv, s: good["fine_cube"](q, k, v, sel, np.ones_like(kv), s))
    elif mutation == "kth_off_by_one":
        # the (k+1)-th and (k+2)-th instead of the k-th and (k+1)-th
        monkeypatch.setattr(O, "kth_gap", lambda s, k: good["kth_gap"](s, min(k + 1, s.shape[-1])))
    elif mutation == "kth_unsorted":
        def bad(scores, k):
            kth = scores[..., k - 1]
            return kth, (scores[..., k] if k < scores.shape[-1] else np.full(kth.shape, -np.inf))
        monkeypatch.setattr(O, "kth_gap", bad)
    elif mutation == "kth_ascending":
        def bad(scores, k):
            s = np.sort(scores, axis=-1)
            kth = s[..., k - 1]
            return kth, (s[..., k] if k < scores.shape[-1] else np.full(kth.shape, -np.inf))
        monkeypatch.setattr(O, "kth_gap", bad)
    elif mutation == "bf16_shift15":
        monkeypatch.setattr(O, "bf16_to_f64", lambda u: (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32)
                                                         << np.uint32(15)).view(np.float32).astype(np.float64))
    elif mutation == "bf16_no_sign":
        monkeypatch.setattr(O, "bf16_to_f64", lambda u: np.abs(good["bf16_to_f64"](u)))
    assert not _pins_pass()
