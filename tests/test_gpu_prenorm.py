"""GPU parity of the pre-attention pass (vsa_qk_norm_rope) against the fp64 oracle.

Bound: the kernel computes in float32 (angles in float64) and rounds once to bf16, so each output
is within half a bf16 unit of the exact value plus the float32 error of the rotation, which is
relative to the rotated pair's magnitude: |gpu - exact| <= 0.5 ulp_bf16(exact) + 4e-6 |pair|.
"""
import math

import numpy as np
import pytest
import torch

import synth
import block_sparse_attention_cube_b200 as vsa
from oracle import prenorm_oracle as R
from oracle import vsa_oracle as O

pytestmark = pytest.mark.gpu


def _dev(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def _host(t):
    return O.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _ulp(x):
    return 2.0 ** (np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -120))) - 7)


def _check(got, exact, what):
    pair = np.sqrt(exact[..., 0::2] ** 2 + exact[..., 1::2] ** 2)
    bound = 0.5 * _ulp(exact) + 4e-6 * np.repeat(pair, 2, axis=-1) + 1e-30
    err = np.abs(got - exact)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside the bound, worst {float((err - bound).max())}"


def _shape(w):
    return vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)


CASES = ["tiny_8x8x8", "padded_7x15x16"]


@pytest.mark.parametrize("name", CASES)
@pytest.mark.parametrize("weights", [True, False])
def test_norm_rope_matches_oracle(name, weights):
    w = synth.WORKLOADS[name]
    x = synth.make_projection_inputs(w)
    s = _shape(w)
    wq, wk = (_dev(x["w_q"]), _dev(x["w_k"])) if weights else (None, None)
    qo, ko = vsa.qk_norm_rope(_dev(x["q_raw"]), _dev(x["k_raw"]), s, wq, wk)
    eq, ek = R.qk_norm_rope(O.bf16_to_f64(x["q_raw"]), O.bf16_to_f64(x["k_raw"]), w.grid,
                            O.bf16_to_f64(x["w_q"]) if weights else None,
                            O.bf16_to_f64(x["w_k"]) if weights else None)
    _check(_host(qo), eq, f"{name} q")
    _check(_host(ko), ek, f"{name} k")


def test_norm_rope_theta_eps_and_in_place():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_projection_inputs(w)
    s = _shape(w)
    q, k = _dev(x["q_raw"]), _dev(x["k_raw"])
    qo, ko = vsa.qk_norm_rope(q, k, s, eps=1e-2, theta=500.0)
    eq, ek = R.qk_norm_rope(O.bf16_to_f64(x["q_raw"]), O.bf16_to_f64(x["k_raw"]), w.grid, eps=1e-2, theta=500.0)
    _check(_host(qo), eq, "q theta=500 eps=1e-2")
    _check(_host(ko), ek, "k theta=500 eps=1e-2")
    qi, ki = vsa.qk_norm_rope(q, k, s, eps=1e-2, theta=500.0, inplace=True)
    assert qi.data_ptr() == q.data_ptr() and ki.data_ptr() == k.data_ptr()
    assert torch.equal(qi.view(torch.int16), qo.view(torch.int16))
    assert torch.equal(ki.view(torch.int16), ko.view(torch.int16))


def test_sequence_parallel_shards_are_bit_identical_to_the_whole():
    w = synth.WORKLOADS["padded_7x15x16"]   # N = 1680 tokens; 3 shards of 600 (120 padding rows)
    s = _shape(w)
    whole = synth.make_projection_inputs(w)
    qw, kw = vsa.qk_norm_rope(_dev(whole["q_raw"]), _dev(whole["k_raw"]), s, _dev(whole["w_q"]), _dev(whole["w_k"]))
    for r in range(3):
        part = synth.make_projection_inputs(w, 600, 600 * r)
        qp, kp = vsa.qk_norm_rope(_dev(part["q_raw"]), _dev(part["k_raw"]), s, _dev(part["w_q"]),
                                  _dev(part["w_k"]), token_offset=600 * r)
        real = min(600, 1680 - 600 * r)
        assert torch.equal(qp[:, :real].view(torch.int16), qw[:, 600 * r:600 * r + real].view(torch.int16))
        assert torch.equal(kp[:, :real].view(torch.int16), kw[:, 600 * r:600 * r + real].view(torch.int16))
        assert not qp[:, real:].view(torch.int16).any() and not kp[:, real:].view(torch.int16).any()


def test_norm_rope_zero_tokens_is_a_no_op():
    w = synth.WORKLOADS["tiny_8x8x8"]
    s = _shape(w)
    q = torch.zeros((1, 0, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    qo, ko = vsa.qk_norm_rope(q, q.clone(), s, out=(torch.empty_like(q), torch.empty_like(q)))
    assert qo.numel() == 0 and ko.numel() == 0


def test_norm_rope_full_480p_sampled_rows():
    """The 480p grid (21x30x52 tokens, 40 heads of 128) at full size, in the launch configuration the
    benchmark times; 300 sampled tokens (incl. the first and the last) checked against the oracle."""
    w = synth.WORKLOADS["wan480p_dense"]
    x = synth.make_inputs(w)
    s = _shape(w)
    wts = synth.make_projection_inputs(synth.custom_workload("w480", 1, 40, 128, (1, 1, 1), 1))
    q, k = _dev(x["q"]), _dev(x["k"])
    qo, ko = vsa.qk_norm_rope(q, k, s, _dev(wts["w_q"]), _dev(wts["w_k"]))
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, w.tokens - 1], rng.integers(0, w.tokens, 298)]))
    qh = _host(qo[:, torch.from_numpy(rows).cuda()])
    kh = _host(ko[:, torch.from_numpy(rows).cuda()])
    for i, g in enumerate(rows):
        eq, ek = R.qk_norm_rope(O.bf16_to_f64(x["q"][:, g:g + 1]), O.bf16_to_f64(x["k"][:, g:g + 1]), w.grid,
                                O.bf16_to_f64(wts["w_q"]), O.bf16_to_f64(wts["w_k"]), token_offset=int(g))
        _check(qh[:, i:i + 1], eq, f"480p q token {g}")
        _check(kh[:, i:i + 1], ek, f"480p k token {g}")


def test_norm_rope_then_attention_matches_oracle():
    """The pass feeding the attention call: GPU norm/rope -> vsa_forward against oracle norm/rope
    (rounded to bf16) -> oracle forward, with the forward call's usual tolerance."""
    w = synth.WORKLOADS["padded_7x15x16"]
    s = _shape(w)
    x = synth.make_projection_inputs(w)
    base = synth.make_inputs(w)
    qo, ko = vsa.qk_norm_rope(_dev(x["q_raw"]), _dev(x["k_raw"]), s, _dev(x["w_q"]), _dev(x["w_k"]))
    scale = 1 / math.sqrt(w.head_dim)
    got = _host(vsa.forward(qo, ko, _dev(base["v"]), s, w.topk, scale, _dev(base["g_coarse"]), _dev(base["g_fine"])))
    eq, ek = R.qk_norm_rope(O.bf16_to_f64(x["q_raw"]), O.bf16_to_f64(x["k_raw"]), w.grid,
                            O.bf16_to_f64(x["w_q"]), O.bf16_to_f64(x["w_k"]))
    rq = O.bf16_to_f64(synth.bf16_bits_torch(torch.from_numpy(eq)))
    rk = O.bf16_to_f64(synth.bf16_bits_torch(torch.from_numpy(ek)))
    ref = O.forward(rq, rk, O.bf16_to_f64(base["v"]), w.grid, w.topk, scale, O.bf16_to_f64(base["g_coarse"]),
                    O.bf16_to_f64(base["g_fine"]))["out"]
    for h in range(w.heads):
        e = got[0, :, h] - ref[0, :, h]
        assert np.abs(e).max() <= 2e-2 and np.linalg.norm(e) <= 5e-3 * np.linalg.norm(ref[0, :, h]), h


def test_sharded_forward_on_one_rank_is_the_plain_call():
    """block_sparse_attention_cube_b200.sharding with one rank: the pre-attention pass at token offset 0
    then the call on every head, bit-identical to calling the two entry points directly."""
    from block_sparse_attention_cube_b200 import sharding as S
    w = synth.WORKLOADS["padded_7x15x16"]
    s = _shape(w)
    x = synth.make_projection_inputs(w)
    base = synth.make_inputs(w)
    q, k, v = _dev(x["q_raw"]), _dev(x["k_raw"]), _dev(base["v"])
    gc, gf = _dev(base["g_coarse"]), _dev(base["g_fine"])
    wq, wk = _dev(x["w_q"]), _dev(x["w_k"])
    scale = 1 / math.sqrt(w.head_dim)
    got = S.sharded_forward(q, k, v, s, w.topk, scale, gc, gf, norm_rope={"w_q": wq, "w_k": wk})
    qn, kn = vsa.qk_norm_rope(q, k, s, wq, wk)
    ref = vsa.forward(qn, kn, v, s, w.topk, scale, gc, gf)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
