"""Host-side checks of the C ABI (no GPU needed).

* the in-tree library loads and exports every function include/vsa.h declares;
* malformed arguments are rejected synchronously with the documented status,
  before anything touches a device.
"""
import ctypes
import os
import re

import pytest

import block_sparse_attention_cube_b200 as vsa
from block_sparse_attention_cube_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA = 1, 2, 3, 4, 5


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "vsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z_0-9]+)\s*\(", text)))


def test_header_and_binding_agree():
    declared = _declared_functions()
    assert len(declared) >= 16
    assert declared == sorted(_lib.SIGNATURES)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings():
    assert vsa.abi_version() == 3
    for code, name in _lib.STATUS_NAMES.items():
        assert _lib.load().vsa_status_string(code).decode() == name


def _shape(b=1, h=2, d=128, grid=(8, 8, 8)):
    return vsa.Shape(b, h, d, grid).c()


def test_shape_info():
    assert vsa.shape_info(vsa.Shape(1, 40, 128, (21, 30, 52))) == (39936, 624)
    assert vsa.shape_info(vsa.Shape(2, 40, 128, (21, 45, 80))) == (92160, 1440)
    assert vsa.shape_info(vsa.Shape(1, 4, 128, (7, 15, 16))) == (2048, 32)


@pytest.mark.parametrize("shape,code", [
    (_shape(b=0), INVALID), (_shape(h=0), INVALID), (_shape(grid=(0, 8, 8)), INVALID),
    (_shape(d=0), INVALID), (_shape(d=96), UNSUPPORTED), (_shape(d=256), UNSUPPORTED),
    (_shape(b=1, h=200, grid=(256, 256, 256)), INVALID),           # more than 2^31 tiled rows
    (_shape(b=300, h=300, grid=(4, 4, 4)), UNSUPPORTED),           # batch*heads above the grid limit
])
def test_shape_errors(shape, code):
    st = vsa.raw_call("vsa_tile", ctypes.byref(shape), ctypes.c_void_p(4096), ctypes.c_void_p(1 << 40), None)
    assert st == code, vsa.last_error()
    assert vsa.last_error()


def test_null_and_misaligned_pointers():
    s = _shape()
    assert vsa.raw_call("vsa_tile", ctypes.byref(s), None, ctypes.c_void_p(4096), None) == INVALID
    assert "x is NULL" in vsa.last_error()
    assert vsa.raw_call("vsa_tile", ctypes.byref(s), ctypes.c_void_p(4104), ctypes.c_void_p(1 << 40), None) == MISALIGNED
    assert vsa.raw_call("vsa_shape_info", None, None, None) == INVALID


def test_fine_fused_steps_need_an_overflow_word():
    """With precomputed steps the fixed-maximum kernel reports overflow in a caller word: no word, no call."""
    s = _shape()
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 32)) for i in range(8)]
    st = vsa.raw_call("vsa_fine_fused", ctypes.byref(s), p[0], p[1], p[2], p[3], 2, None, p[4], 0.125,
                      None, None, None, p[5], None, None)
    assert st == INVALID and "overflow word" in vsa.last_error()
    st = vsa.raw_call("vsa_fine_fused", ctypes.byref(s), p[0], p[1], p[2], p[3], 2, None, p[4], 0.125,
                      None, None, None, p[5], ctypes.c_void_p(p[6].value + 4), None)
    assert st == MISALIGNED and "overflow" in vsa.last_error()
    # dense attention (idx NULL) runs on the same fixed-maximum kernel: it needs the word too
    st = vsa.raw_call("vsa_fine_fused", ctypes.byref(s), p[0], p[1], p[2], None, 0, None, None, 0.125,
                      None, None, None, p[5], None, None)
    assert st == INVALID and "dense attention without an overflow word" in vsa.last_error()


def test_forward_rerun_argument_checks():
    s = _shape()
    r = ctypes.c_int32(-5)
    ws = ctypes.c_void_p(1 << 40)
    assert vsa.raw_call("vsa_forward_rerun", ctypes.byref(s), 2, 1, ws, None, None) == INVALID
    assert vsa.raw_call("vsa_forward_rerun", ctypes.byref(s), 0, 1, ws, ctypes.byref(r), None) == INVALID
    assert vsa.raw_call("vsa_forward_rerun", ctypes.byref(s), 2, 1, None, ctypes.byref(r), None) == INVALID
    # a sparse call with more cubes than the precomputed schedule holds (32,000: its per-warp marks
    # exceed 48 KB of shared memory) walks the selection itself with online rescaling: no fixed-maximum
    # stage ran, so the answer comes without touching the device
    big = _shape(grid=(80, 160, 160))
    assert vsa.raw_call("vsa_forward_rerun", ctypes.byref(big), 2, 0, ws, ctypes.byref(r), None) == 0
    assert r.value == 0


def test_coarse_workspace_checks():
    s = _shape()
    need = vsa.raw_call("vsa_coarse_workspace_bytes", ctypes.byref(s))
    # three float32 inputs as three bf16 parts each, and 8 bytes of softmax statistics per score row
    up = lambda n: (n + 255) // 256 * 256
    assert need == 3 * up(3 * 2 * 8 * 128 * 2) + up(2 * 8 * 8)
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 32)) for i in range(6)]
    call = lambda ws, n: vsa.raw_call("vsa_coarse", ctypes.byref(s), p[0], p[1], p[2], 0.125, p[3], p[4], ws, n, None)
    assert call(None, need) == WORKSPACE
    assert call(p[5], need - 1) == WORKSPACE
    assert call(ctypes.c_void_p(p[5].value + 16), need) == MISALIGNED


def test_overlapping_input_and_output_rejected():
    s = _shape()
    base = 1 << 40
    st = vsa.raw_call("vsa_tile", ctypes.byref(s), ctypes.c_void_p(base), ctypes.c_void_p(base + 1024), None)
    assert st == INVALID and "overlaps" in vsa.last_error()


@pytest.mark.parametrize("k", [0, -1, 9])
def test_topk_out_of_range(k):
    s = _shape()   # 8 cubes
    st = vsa.raw_call("vsa_topk", ctypes.byref(s), ctypes.c_void_p(1 << 40), k, ctypes.c_void_p(1 << 41), None)
    assert st == INVALID and "top-k" in vsa.last_error()


@pytest.mark.parametrize("scale", [0.0, -1.0, float("inf"), float("nan")])
def test_bad_scale(scale):
    s = _shape()
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 32)) for i in range(5)]
    st = vsa.raw_call("vsa_fine", ctypes.byref(s), p[0], p[1], p[2], None, 0, None, scale, p[3], None, None)
    assert st == INVALID and "scale" in vsa.last_error()


def test_workspace_checks():
    s = _shape()
    need = vsa.raw_call("vsa_workspace_bytes", ctypes.byref(s), 2)
    assert need > 0
    assert vsa.raw_call("vsa_workspace_bytes", ctypes.byref(s), 0) == 0
    assert vsa.raw_call("vsa_workspace_bytes", ctypes.byref(s), 9) == 0
    assert vsa.raw_call("vsa_workspace_bytes_host", ctypes.byref(s), 2) > need
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 32)) for i in range(6)]
    args = (ctypes.byref(s), p[0], p[1], p[2], None, None, 2, 0.125)
    assert vsa.raw_call("vsa_forward", *args, None, need, p[3], None) == WORKSPACE
    assert vsa.raw_call("vsa_forward", *args, p[4], need - 1, p[3], None) == WORKSPACE
    assert vsa.raw_call("vsa_forward", *args, ctypes.c_void_p(p[4].value + 16), need, p[3], None) == MISALIGNED


def test_workspace_size_480p_matches_layout():
    # Q, K, V are read in place, so the workspace holds the pooled q, k, v as three bf16 parts each
    # (3 x 3 x 624*40*128*2 B), the per-row softmax statistics (624*40*8 B), o_coarse (624*40*128*4 B),
    # the scores (624*624*40*4 B), idx (624*40*32*4 B) and the work order (624*40*4 B) with its
    # signatures (624*40*8 B), the fine stage's steps and its overflow word, each rounded up to 256 B
    s = vsa.Shape(1, 40, 128, (21, 30, 52)).c()
    up = lambda n: (n + 255) // 256 * 256
    coarse = 3 * up(3 * 624 * 40 * 128 * 2) + up(624 * 40 * 8) + up(624 * 40 * 128 * 4) + up(624 * 624 * 40 * 4)
    expect = coarse + up(624 * 40 * 32 * 4) + up(624 * 40 * 4) + up(624 * 40 * 8) \
        + up(312 * 40 * 32 * 8) \
        + up(8)   # work-order signatures; steps: 312 pairs of query cubes x k steps x 8 B; overflow pair
    assert vsa.raw_call("vsa_workspace_bytes", ctypes.byref(s), 32) == expect
    # every cube selected: dense attention; the coarse buffers are for a coarse gate only
    assert vsa.raw_call("vsa_workspace_bytes", ctypes.byref(s), 624) == coarse + up(8)


def test_probe_limit_checked_before_device():
    assert vsa.raw_call("vsa_debug_wait_probe", 10, None) == INVALID
    assert vsa.raw_call("vsa_debug_wait_probe", 10**12, None) == INVALID


def test_group_limits_checked_before_device():
    s = vsa.Shape(1, 2, 128, (40, 40, 44)).c()     # 10*10*11 = 1100 cubes: fine
    big = vsa.Shape(1, 2, 128, (80, 80, 44)).c()   # 20*20*11 = 4400 cubes: above the grouping limit
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 34)) for i in range(2)]
    assert vsa.raw_call("vsa_group", ctypes.byref(big), p[0], p[1], None) == UNSUPPORTED
    assert vsa.raw_call("vsa_group", ctypes.byref(s), None, p[1], None) == INVALID


def _norm_rope_call(s, q, k, wq, wk, eps, theta, off, n, qo, ko):
    return vsa.raw_call("vsa_qk_norm_rope", ctypes.byref(s), q, k, wq, wk, ctypes.c_float(eps), ctypes.c_float(theta),
                        ctypes.c_int64(off), ctypes.c_int64(n), qo, ko, None)


def _far(i):
    return ctypes.c_void_p((1 << 40) + i * (1 << 32))


@pytest.mark.parametrize("eps, theta, off, n, word", [
    (0.0, 1e4, 0, 512, "eps"), (-1.0, 1e4, 0, 512, "eps"), (float("nan"), 1e4, 0, 512, "eps"),
    (float("inf"), 1e4, 0, 512, "eps"), (1e-6, 1.0, 0, 512, "theta"), (1e-6, float("nan"), 0, 512, "theta"),
    (1e-6, 1e4, -1, 512, "token_offset"), (1e-6, 1e4, 0, -5, "n_tokens")])
def test_norm_rope_bad_scalars(eps, theta, off, n, word):
    s = _shape()
    st = _norm_rope_call(s, _far(0), _far(1), None, None, eps, theta, off, n, _far(2), _far(3))
    assert st == INVALID and word in vsa.last_error()


def test_norm_rope_pointer_checks():
    s = _shape()
    assert _norm_rope_call(s, None, _far(1), None, None, 1e-6, 1e4, 0, 8, _far(2), _far(3)) == INVALID
    assert _norm_rope_call(s, _far(0), _far(1), ctypes.c_void_p((1 << 40) + 8), None, 1e-6, 1e4, 0, 8, _far(2),
                           _far(3)) == MISALIGNED
    # outputs may not overlap another tensor (only q_out == q and k_out == k are allowed)
    st = _norm_rope_call(s, _far(0), _far(1), None, None, 1e-6, 1e4, 0, 8, _far(1), _far(3))
    assert st == INVALID and "overlap" in vsa.last_error()
    st = _norm_rope_call(s, _far(0), _far(1), None, None, 1e-6, 1e4, 0, 8, _far(2), _far(2))
    assert st == INVALID and "overlap" in vsa.last_error()
    st = _norm_rope_call(s, _far(0), _far(1), None, None, 1e-6, 1e4, 0, 8, _far(0), _far(0))
    assert st == INVALID and "overlap" in vsa.last_error()


def test_norm_rope_row_width_limit():
    s = vsa.Shape(1, 65, 128, (4, 4, 4)).c()   # H*D = 8320 > 8192
    st = _norm_rope_call(s, _far(0), _far(1), None, None, 1e-6, 1e4, 0, 64, _far(2), _far(3))
    assert st == UNSUPPORTED and "H*D" in vsa.last_error()
