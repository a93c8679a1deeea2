"""vsa_forward_noalloc: the whole call for callers that cannot allocate device memory.

Such callers (a plugin handed only its input and output buffers, a runtime
whose pool owns the device, real-time code that must not allocate after
start-up) get the same result as vsa_forward with a caller workspace; the
workspace lives in the library's static device array instead.  The test
goes through the C ABI (ctypes) and compares two calls in a row, of different
shapes and in both orders, with the existing entry point, bit for bit.  The
file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_cube_b200 as vsa
import synth
from block_sparse_attention_cube_b200 import _lib
from tests._util import to_dev

WORKSPACE = 4   # VSA_ERR_WORKSPACE


def _c_call(w, d, out):
    lib = _lib.load()
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    st = lib.vsa_forward_noalloc(ctypes.byref(s.c()), ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g_coarse"]),
                                 ptr(d["g_fine"]), w.topk, 1.0 / np.sqrt(w.head_dim), ptr(out),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.vsa_last_error().decode()


def _two_calls_in_a_row(names, device):
    """Each shape through the static workspace and through vsa_forward with a caller workspace: the same
    kernels on the same inputs, so the bits must agree exactly."""
    with torch.cuda.device(device):
        results = []
        for name in names:
            w = synth.WORKLOADS[name]
            assert vsa.workspace_bytes(vsa.Shape(w.batch, w.heads, w.head_dim, w.grid), w.topk) \
                <= vsa.NOALLOC_WORKSPACE_BYTES
            d = {k: to_dev(v).to(device) for k, v in synth.make_inputs(w).items()}
            out = torch.empty_like(d["q"])
            _c_call(w, d, out)
            ref = vsa.forward(d["q"], d["k"], d["v"], vsa.Shape(w.batch, w.heads, w.head_dim, w.grid), w.topk,
                              1.0 / np.sqrt(w.head_dim), d["g_coarse"], d["g_fine"])
            torch.cuda.synchronize()
            results.append((name, out, ref))
        vsa.device_status()
        for name, got, ref in results:
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"{name}: noalloc differs from forward"


@pytest.mark.gpu
@pytest.mark.parametrize("names", [("padded_7x15x16", "tiny_8x8x8"), ("tiny_8x8x8", "padded_7x15x16")],
                         ids=["large_then_small", "small_then_large"])
def test_noalloc_matches_forward_on_two_calls_in_a_row(names):
    _two_calls_in_a_row(names, torch.device("cuda", 0))


@pytest.mark.gpu
def test_noalloc_on_a_second_device():
    """The static array's address is looked up per device: a call on the second GPU uses that GPU's copy."""
    if torch.cuda.device_count() < 2:
        pytest.skip("one GPU visible")
    _two_calls_in_a_row(("tiny_8x8x8", "padded_7x15x16"), torch.device("cuda", 1))


def test_noalloc_rejects_shapes_beyond_the_static_workspace():
    s = vsa.Shape(1, 40, 128, (21, 30, 52))
    need = vsa.workspace_bytes(s, 32)
    assert need > vsa.NOALLOC_WORKSPACE_BYTES
    p = [ctypes.c_void_p((1 << 40) + i * (1 << 34)) for i in range(4)]
    st = vsa.raw_call("vsa_forward_noalloc", ctypes.byref(s.c()), p[0], p[1], p[2], None, None, 32, 0.125, p[3], None)
    assert st == WORKSPACE
    msg = vsa.last_error()
    assert "static workspace" in msg and str(need) in msg
