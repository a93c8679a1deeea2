"""Pins for the fp64 oracle of the pre-attention pass (Q/K RMSNorm + 3D RoPE).

Checked against things other than the oracle itself:
* a library routine the norm reduces to (torch.nn.functional.rms_norm, fp64);
* the rotation written as complex multiplication (numpy complex128), an
  independent path for the pair order and the sign of the turn;
* properties any rotary embedding must have: identity at the origin, norm
  preserved per pair, dot products that depend on positions only through
  their difference, angles linear in the position, each axis moving only its
  own band of pairs;
* closed forms of RMSNorm (mean square of the output, scale invariance);
* shard equivalence (sequence-parallel token offsets and padding rows);
* planted mistakes in the oracle that these pins must catch.
"""
import numpy as np
import pytest
import torch

from oracle import prenorm_oracle as R


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# the reading of the band split (t first, x and y floor(D/6) pairs each), fixed here independently
BANDS = {128: (22, 21, 21), 64: (12, 10, 10)}


@pytest.mark.parametrize("D", [128, 64])
def test_band_sizes_cover_every_pair(D):
    assert R.rope_bands(D) == BANDS[D]
    assert sum(R.rope_bands(D)) == D // 2


# ---------------------------------------------------------------- RMSNorm
def test_rms_norm_equals_library():
    x = _rand((3, 7, 5120), 1) * 3.0
    w = _rand((5120,), 2)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (5120,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(R.rms_norm(x, w, 1e-6), ref, rtol=1e-13, atol=1e-13)


def test_rms_norm_closed_forms():
    x = _rand((4, 256), 3) * np.array([[0.01], [1.0], [30.0], [1e-3]])
    eps = 1e-6
    y = R.rms_norm(x, None, eps)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12)
    # without eps the result ignores a positive scale of the input
    np.testing.assert_allclose(R.rms_norm(7.5 * x, None, 0.0), R.rms_norm(x, None, 0.0), rtol=1e-12)
    # the weight multiplies channel by channel
    w = _rand((256,), 4)
    np.testing.assert_allclose(R.rms_norm(x, w, eps), y * w, rtol=1e-13)


# ---------------------------------------------------------------- RoPE
@pytest.mark.parametrize("D", [64, 128])
def test_rope_equals_complex_multiplication(D):
    n, H = 11, 3
    x = _rand((n, H, D), 5)
    coords = np.random.default_rng(6).integers(0, 60, size=(n, 3))
    ang = R.rope_angles(coords, D)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)[:, None, :]
    got = R.rope_apply(x, ang)
    np.testing.assert_allclose(got[..., 0::2], z.real, atol=1e-12)
    np.testing.assert_allclose(got[..., 1::2], z.imag, atol=1e-12)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_identity_at_origin_and_norm_per_pair(D):
    x = _rand((5, 2, D), 7)
    np.testing.assert_array_equal(R.rope_apply(x, R.rope_angles(np.zeros((5, 3), np.int64), D)), x)
    coords = np.random.default_rng(8).integers(0, 80, size=(5, 3))
    y = R.rope_apply(x, R.rope_angles(coords, D))
    np.testing.assert_allclose(y[..., 0::2] ** 2 + y[..., 1::2] ** 2, x[..., 0::2] ** 2 + x[..., 1::2] ** 2,
                               rtol=1e-12)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_dot_products_depend_on_relative_position(D):
    rng = np.random.default_rng(9)
    q, k = _rand((1, 1, D), 10), _rand((1, 1, D), 11)
    for _ in range(20):
        p1, p2, shift = (rng.integers(0, 50, size=(1, 3)) for _ in range(3))
        def dot(a, b):
            return float(np.sum(R.rope_apply(q, R.rope_angles(a, D)) * R.rope_apply(k, R.rope_angles(b, D))))
        assert abs(dot(p1 + shift, p2 + shift) - dot(p1, p2)) < 1e-10


@pytest.mark.parametrize("D", [64, 128])
def test_rope_angles_linear_in_position_with_unit_first_frequency(D):
    a, b = np.array([[3, 5, 7]]), np.array([[10, 1, 4]])
    np.testing.assert_allclose(R.rope_angles(a + b, D), R.rope_angles(a, D) + R.rope_angles(b, D), rtol=1e-14)
    one = R.rope_angles(np.eye(3, dtype=np.int64), D)   # unit step along t, x, y
    start = 0
    for axis, p in enumerate(R.rope_bands(D)):
        band = one[axis, start:start + p]
        assert band[0] == 1.0                       # the band's first pair turns one radian per position
        ratios = band[1:] / band[:-1]               # then a geometric fall towards theta^-1
        np.testing.assert_allclose(ratios, ratios[0], rtol=1e-12)
        assert 0.0 < band[-1] < 1.0
        start += p


@pytest.mark.parametrize("D", [64, 128])
def test_each_axis_moves_only_its_band(D):
    x = _rand((1, 1, D), 12)
    base = R.rope_apply(x, R.rope_angles(np.array([[2, 3, 4]]), D))
    pt, px, py = BANDS[D]
    edges = [0, pt, pt + px, pt + px + py]
    for axis in range(3):
        c = np.array([[2, 3, 4]])
        c[0, axis] += 5
        moved = R.rope_apply(x, R.rope_angles(c, D))
        changed = np.abs(moved - base).reshape(D // 2, 2).max(axis=1) > 1e-12
        expect = np.zeros(D // 2, bool)
        expect[edges[axis]:edges[axis + 1]] = True
        np.testing.assert_array_equal(changed, expect)


def test_token_coords_follow_the_token_order():
    grid = (3, 4, 5)
    coords = R.token_coords(np.arange(60), grid)
    t, x, y = np.meshgrid(np.arange(3), np.arange(4), np.arange(5), indexing="ij")
    np.testing.assert_array_equal(coords, np.stack([t.ravel(), x.ravel(), y.ravel()], axis=1))


# ---------------------------------------------------------------- the whole pass
def test_norm_rope_is_norm_then_rotation_per_head():
    grid = (2, 3, 4)
    B, H, D = 2, 3, 64
    x = _rand((B, 24, H, D), 13)
    w = _rand((H * D,), 14)
    got = R.norm_rope(x, grid, w, 1e-6, 10000.0)
    ang = R.rope_angles(R.token_coords(np.arange(24), grid), D)
    for b in range(B):
        y = R.rms_norm(x[b].reshape(24, H * D), w, 1e-6).reshape(24, H, D)
        np.testing.assert_allclose(got[b], R.rope_apply(y, ang), rtol=1e-13, atol=1e-13)


def test_sequence_parallel_shards_equal_the_whole_and_padding_is_zero():
    grid = (3, 5, 7)   # N = 105 tokens, 4 shards of 27 (3 padding rows at the end)
    B, H, D = 1, 2, 128
    N = 105
    x = _rand((B, 108, H, D), 15)
    whole = R.norm_rope(x[:, :N], grid)
    for r in range(4):
        part = R.norm_rope(x[:, 27 * r:27 * (r + 1)], grid, token_offset=27 * r)
        real = min(27, N - 27 * r)
        np.testing.assert_allclose(part[:, :real], whole[:, 27 * r:27 * r + real], rtol=1e-13, atol=1e-13)
        assert not part[:, real:].any()


# ---------------------------------------------------------------- planted mistakes
def _pins():
    for D in (64, 128):
        test_band_sizes_cover_every_pair(D)
    test_rms_norm_equals_library()
    test_rms_norm_closed_forms()
    for D in (64, 128):
        test_rope_equals_complex_multiplication(D)
        test_rope_identity_at_origin_and_norm_per_pair(D)
        test_rope_dot_products_depend_on_relative_position(D)
        test_rope_angles_linear_in_position_with_unit_first_frequency(D)
        test_each_axis_moves_only_its_band(D)
    test_token_coords_follow_the_token_order()
    test_norm_rope_is_norm_then_rotation_per_head()


def _bad_rope_sign(x, angles):
    a, b = x[..., 0::2], x[..., 1::2]
    c, s = np.cos(angles)[:, None, :], np.sin(angles)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = a * c + b * s
    out[..., 1::2] = -a * s + b * c
    return out


def _bad_rope_pairs(x, angles):
    # rotates channel d with channel d + D/2 instead of its neighbour
    D = x.shape[-1]
    a, b = x[..., :D // 2], x[..., D // 2:]
    c, s = np.cos(angles)[:, None, :], np.sin(angles)[:, None, :]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _bad_bands(D):
    pt, px, py = (D // 2 - 2 * (D // 6), D // 6, D // 6)
    return px, pt, py


def _bad_angles_offset(coords, head_dim, theta=R.DEFAULT_THETA):
    coords = np.asarray(coords, dtype=np.float64) + 1.0
    cols = []
    for axis, p in enumerate(R.rope_bands(head_dim)):
        cols.append(coords[:, axis:axis + 1] * theta ** (-np.arange(p) / p)[None, :])
    return np.concatenate(cols, axis=1)


def _bad_rms(x, w, eps=R.DEFAULT_EPS):
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if w is None else y + w


def _bad_coords(n, grid):
    T, X, Y = grid
    n = np.asarray(n, dtype=np.int64)
    return np.stack([n // (X * Y), n % X, (n // X) % Y], axis=-1)


def test_pins_pass_on_the_oracle():
    _pins()


@pytest.mark.parametrize("mutation", [
    ("rope_apply", _bad_rope_sign), ("rope_apply", _bad_rope_pairs), ("rope_bands", _bad_bands),
    ("rope_angles", _bad_angles_offset), ("rms_norm", _bad_rms), ("token_coords", _bad_coords)])
def test_planted_mistake_is_caught(monkeypatch, mutation):
    name, fn = mutation
    monkeypatch.setattr(R, name, fn)
    with pytest.raises(AssertionError):
        _pins()
