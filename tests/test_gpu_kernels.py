"""GPU parity of every step of the path against the fp64 oracle, on sizes the
oracle runs in full (several cubes, padded and unpadded grids, ragged pairs)
and on the edge cases of the method."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cube_b200 as vsa
import synth
from oracle import vsa_oracle as O
from tests._util import (COARSE_REL_L2, LSE_ABS, assert_selection, bf16_bits, check_close, check_heads, from_dev,
                         to_dev)

pytestmark = pytest.mark.gpu

SMALL = ["tiny_8x8x8", "tiny_8x8x8_all", "padded_7x15x16"]
EDGE_SHAPES = {
    # name: (batch, heads, head_dim, grid, topk)
    "odd_cubes_4x4x12": (1, 3, 128, (4, 4, 12), 2),       # C = 3: last pair has one cube
    "single_cube_3x2x4": (1, 2, 128, (3, 2, 4), 1),       # C = 1, partial cube
    "ragged_9x6x5_d64": (2, 2, 64, (9, 6, 5), 4),         # B = 2, d = 64, partial cubes on every axis
    "wide_5x9x30": (1, 2, 128, (5, 9, 30), 7),            # C = 2*3*8 = 48, odd k
}


def _workload(name):
    if name in synth.WORKLOADS:
        return synth.WORKLOADS[name]
    b, h, d, grid, k = EDGE_SHAPES[name]
    return synth.custom_workload(name, b, h, d, grid, k, field=True, wid=91 + list(EDGE_SHAPES).index(name))


def _shape(w):
    return vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)


@pytest.fixture(scope="module", params=SMALL + list(EDGE_SHAPES))
def case(request):
    w = _workload(request.param)
    x = synth.make_inputs(w)
    dev = {k: to_dev(v) for k, v in x.items()}
    f64 = {k: O.bf16_to_f64(v) for k, v in x.items()}
    return w, x, dev, f64


def test_tile_bit_exact_and_roundtrip(case):
    w, x, dev, _ = case
    s = _shape(w)
    for name in ("q", "k", "v"):
        xt = vsa.tile(dev[name], s)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(xt), O.tile(x[name], w.grid)), name
        back = vsa.untile(xt, s)
        assert np.array_equal(bf16_bits(back), x[name]), name


def test_pool_matches_oracle(case):
    w, _, dev, f64 = case
    s = _shape(w)
    for name in ("q", "k", "v"):
        got = from_dev(vsa.pool(vsa.tile(dev[name], s), s))
        ref = O.pool(O.tile(f64[name], w.grid), w.grid)
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)


def test_coarse_on_shared_inputs(case):
    """vsa_coarse on float32 pooled vectors the test generates, against the oracle's coarse step."""
    w, _, _, f64 = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    bars32 = [O.pool(O.tile(f64[n], w.grid), w.grid).astype(np.float32) for n in ("q", "k", "v")]
    scores, oc = vsa.coarse(*(torch.from_numpy(b).cuda() for b in bars32), s, scale)
    r_scores, r_oc = O.coarse(*(b.astype(np.float64) for b in bars32), scale)
    g_scores, g_oc = from_dev(scores), from_dev(oc)
    np.testing.assert_allclose(g_scores, r_scores, rtol=0, atol=1e-5 * max(1.0, np.abs(r_scores).max()))
    assert np.linalg.norm(g_oc - r_oc) / np.linalg.norm(r_oc) <= COARSE_REL_L2


def test_topk_bit_exact_on_shared_scores(case):
    """vsa_topk on float32 score arrays the test generates (many exact ties, signed zeros)."""
    w = case[0]
    s = _shape(w)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(11)
    shape = (w.batch, w.heads, C, C)
    arrays = [rng.integers(-3, 4, size=shape).astype(np.float32),
              (rng.standard_normal(shape) * 0.1).astype(np.float32),
              np.where(rng.random(shape) < 0.5, np.float32(-0.0), np.float32(0.0))]
    for a in arrays:
        for k in sorted({1, w.topk, C}):
            g = vsa.topk(torch.from_numpy(a).cuda(), s, k).cpu().numpy()
            assert np.array_equal(g, O.topk(a.astype(np.float64), k)), k


def test_selection_matches_oracle(case):
    """The GPU's own pool -> coarse -> top-k against the oracle's, up to documented near-ties."""
    w, _, dev, f64 = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    bars = [vsa.pool(vsa.tile(dev[n], s), s) for n in ("q", "k", "v")]
    scores, oc = vsa.coarse(*bars, s, scale)
    g_idx = vsa.topk(scores, s, w.topk).cpu().numpy()
    ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk)
    assert_selection(g_idx, ora["idx"], ora["scores"], w.topk, f"{w.name} selection")
    np.testing.assert_allclose(from_dev(scores), ora["scores"], rtol=0,
                               atol=1e-5 * max(1.0, np.abs(ora["scores"]).max()))
    rel = np.linalg.norm(from_dev(oc) - ora["o_coarse"]) / np.linalg.norm(ora["o_coarse"])
    assert rel <= COARSE_REL_L2, rel


def test_fine_sparse_matches_oracle(case):
    """The fine kernel on the oracle's own selection against the oracle's fine step."""
    w, _, dev, f64 = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, scale)
    qt, kt, vt = (vsa.tile(dev[n], s) for n in ("q", "k", "v"))
    o, lse = vsa.fine(qt, kt, vt, s, torch.from_numpy(ora["idx"]).cuda(), scale)
    check_heads(from_dev(o), ora["o_fine"], w.grid, "o_fine")
    valid = O.key_valid_mask(w.grid)
    err = np.abs(from_dev(lse)[:, :, valid] - ora["lse"][:, :, valid]).max()
    assert err <= LSE_ABS, err


def test_dense_matches_oracle(case):
    w, _, dev, f64 = case
    s = _shape(w)
    qt, kt, vt = (vsa.tile(dev[n], s) for n in ("q", "k", "v"))
    o, lse = vsa.fine(qt, kt, vt, s, None)
    out = from_dev(vsa.untile(o, s))
    r_out, r_lse = O.dense(f64["q"], f64["k"], f64["v"], w.grid)
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(out[b, :, h], r_out[b, :, h], f"dense[b={b},h={h}]")
    g_lse = from_dev(lse)
    g_lse_tok = O.untile(g_lse[..., None], w.grid)[..., 0]
    assert np.abs(g_lse_tok - r_lse).max() <= LSE_ABS
    # the whole call with top-k = C and no gates: dense attention over blocks of
    # 64 consecutive real tokens read in place (no tiling, no padding)
    npad, C = vsa.shape_info(s)
    out2 = from_dev(vsa.forward(dev["q"], dev["k"], dev["v"], s, C))
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(out2[b, :, h], r_out[b, :, h], f"dense forward[b={b},h={h}]")


def test_forward_matches_the_stages_run_one_by_one(case):
    """vsa_forward (pool read in place, cube gathers, merge in the fine epilogue) against
    tile -> pool -> coarse -> top-k -> group -> fine -> combine -> untile through the
    per-step entry points.  The selections are identical (the same float32 pooling order);
    the outputs differ only by the bf16 rounding of O_f that the staged path makes."""
    w, _, dev, _ = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    gc, gf = dev["g_coarse"], dev["g_fine"]
    qt, kt, vt = (vsa.tile(dev[n], s) for n in ("q", "k", "v"))
    bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
    scores, oc = vsa.coarse(*bars, s, scale)
    idx = vsa.topk(scores, s, w.topk)
    order = vsa.group(scores, s)
    of, _ = vsa.fine(qt, kt, vt, s, idx, scale, order=order)
    staged = from_dev(vsa.untile(vsa.combine(oc, of, s, gc, gf), s))
    fused = from_dev(vsa.forward(dev["q"], dev["k"], dev["v"], s, w.topk, scale, gc, gf))
    assert np.array_equal(vsa.topk(vsa.coarse(*[vsa.pool(t, s) for t in (qt, kt, vt)], s, scale)[0], s,
                                   w.topk).cpu().numpy(), idx.cpu().numpy())
    # the forward call walks its steps in a different order (precomputed, grouped by the tiles
    # that use them; dense attention over blocks of consecutive real tokens), a different but
    # equally valid summation order, so the oracle tolerance applies
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(fused[b, :, h], staged[b, :, h], f"forward vs stages[b={b},h={h}]")
    # with the fine kernel's own walk (no precomputed steps) the two paths share every step,
    # so they differ by at most the staged path's extra rounding of O_f (half a bf16 unit of
    # O_f, times g_f <= 1) plus one unit of the result (the two final roundings)
    _, C = vsa.shape_info(s)
    if w.topk == C:
        return
    walk = from_dev(vsa.fine_fused(dev["q"], dev["k"], dev["v"], s, idx, scale, order, oc, gc, gf))
    ulp = lambda a: 2.0 ** (np.floor(np.log2(np.maximum(np.abs(a), 2.0 ** -100))) - 7)
    of_tok = from_dev(vsa.untile(of, s))
    bound = ulp(staged) + 0.5 * ulp(of_tok) + 1e-6
    assert np.all(np.abs(walk - staged) <= bound), "fused fine stage differs from the staged path beyond rounding"


def _compare_call(w, dev, f64, k, scale, gates=True):
    """The whole call against the oracle's.  The GPU selection must equal the oracle's up to
    documented near-ties (counted); the oracle's fine stage then runs over the GPU's selection, so
    every real token is compared, a near-tie swap included."""
    s = _shape(w)
    gc, gf = (dev["g_coarse"], dev["g_fine"]) if gates else (None, None)
    out = vsa.forward(dev["q"], dev["k"], dev["v"], s, k, scale, gc, gf)
    bars = [vsa.pool(vsa.tile(dev[n], s), s) for n in ("q", "k", "v")]
    g_idx = vsa.topk(vsa.coarse(*bars, s, scale)[0], s, k).cpu().numpy()
    args = (f64["q"], f64["k"], f64["v"], w.grid, k, scale,
            f64["g_coarse"] if gates else None, f64["g_fine"] if gates else None)
    ora = O.forward(*args)
    r = assert_selection(g_idx, ora["idx"], ora["scores"], k, f"{w.name} forward k={k}")
    if r.differ:
        ora = O.forward(*args, idx_override=g_idx)
    got = from_dev(out)
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(got[b, :, h], ora["out"][b, :, h], f"out[b={b},h={h}] k={k}")


@pytest.mark.parametrize("grid,k", [((4, 4, 8400), 4), ((4, 4, 16800), 3)], ids=["C2100", "C4200"])
def test_forward_beyond_the_register_selection(grid, k):
    """More cubes than the register-resident selection takes (C > 2048: the shared-memory top-k kernel, the
    work order from vsa_group, the coarse output's softmax statistics from their own pass) and than the
    work-order sort takes (C > 4096: no grouping): the whole gated call against the oracle."""
    w = synth.custom_workload(f"long_{grid[2]}", 1, 1, 64, grid, k, field=True, wid=95 + grid[2] // 8400)
    x = synth.make_inputs(w)
    dev = {n: to_dev(v) for n, v in x.items()}
    f64 = {n: O.bf16_to_f64(v) for n, v in x.items()}
    _, C = vsa.shape_info(_shape(w))
    assert C > 2048
    _compare_call(w, dev, f64, k, 1 / math.sqrt(64))


def test_forward_matches_oracle(case):
    w, _, dev, f64 = case
    _compare_call(w, dev, f64, w.topk, 1 / math.sqrt(w.head_dim))


def test_forward_without_gates_matches_oracle(case):
    """Both gates NULL (g_c = 0, g_f = 1): the call skips the coarse output, which only the merge uses."""
    w, _, dev, f64 = case
    _compare_call(w, dev, f64, w.topk, 1 / math.sqrt(w.head_dim), gates=False)


def test_combine_matches_oracle(case):
    w, _, dev, f64 = case
    s = _shape(w)
    rng = np.random.default_rng(5)
    npad, C = vsa.shape_info(s)
    oc = torch.from_numpy(rng.normal(size=(w.batch, w.heads, C, w.head_dim)).astype(np.float32)).cuda()
    of_bits = synth.f32_to_bf16_bits(rng.normal(size=(w.batch, w.heads, npad, w.head_dim)).astype(np.float32))
    of = to_dev(of_bits)
    for gc, gf in ((dev["g_coarse"], dev["g_fine"]), (None, None), (dev["g_coarse"], None)):
        got = from_dev(vsa.combine(oc, of, s, gc, gf))
        ref = O.combine(oc.cpu().numpy().astype(np.float64), O.bf16_to_f64(of_bits),
                        None if gc is None else f64["g_coarse"], None if gf is None else f64["g_fine"], w.grid)
        # one bf16 rounding of a float32 value
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-6)


# ---------------------------------------------------------------- edge cases
def _run_fine(w, x, idx=None, scale=None):
    s = _shape(w)
    d = {k: to_dev(v) for k, v in x.items()}
    qt, kt, vt = (vsa.tile(d[n], s) for n in ("q", "k", "v"))
    return qt, kt, vt, s


def test_zero_query_selects_first_cubes_and_averages_values():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    x["q"] = np.zeros_like(x["q"])
    qt, kt, vt, s = _run_fine(w, x)
    bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
    scores, _ = vsa.coarse(*bars, s)
    idx = vsa.topk(scores, s, 5)
    first5 = np.broadcast_to(np.arange(5, dtype=np.int32), idx.shape)
    assert np.array_equal(idx.cpu().numpy(), first5)
    o, lse = vsa.fine(qt, kt, vt, s, idx)
    r_o, r_lse = O.fine(*(O.tile(O.bf16_to_f64(x[n]), w.grid) for n in ("q", "k", "v")), first5,
                        1 / math.sqrt(128), w.grid)
    check_heads(from_dev(o), r_o, w.grid, "o_fine(q=0)")


def test_constant_values_give_ones():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    x["v"] = np.full_like(x["v"], 0x3F80)   # bf16 1.0
    qt, kt, vt, s = _run_fine(w, x)
    o, _ = vsa.fine(qt, kt, vt, s, None)
    got = from_dev(o)[:, :, O.key_valid_mask(w.grid)]
    assert np.abs(got - 1.0).max() <= 2 ** -8


def test_overflow_scores_stay_finite():
    """q.k/sqrt(d) near 150-200: an unshifted fp32 exp overflows; the online softmax must not."""
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    for n in ("q", "k"):
        x[n] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(x[n]) * 16.0)
    f64 = {k: O.bf16_to_f64(v) for k, v in x.items()}
    qt, kt, vt, s = _run_fine(w, x)
    o, lse = vsa.fine(qt, kt, vt, s, None)
    r_o, r_lse = O.fine(*(O.tile(f64[n], w.grid) for n in ("q", "k", "v")), None, 1 / math.sqrt(128), w.grid)
    valid = O.key_valid_mask(w.grid)
    assert r_lse[:, :, valid].max() > 100
    check_heads(from_dev(o), r_o, w.grid, "o_fine(overflow)")
    assert np.abs(from_dev(lse)[:, :, valid] - r_lse[:, :, valid]).max() <= LSE_ABS


@pytest.mark.parametrize("dense", [False, True])
def test_overflow_scores_through_the_forward_call(dense):
    """The fused call on the same scaled inputs.  Sparse: the one-tile kernel's fixed per-row maxima
    overflow, it raises its overflow word and the call re-runs the fine stage with the online
    rescaling kernel; the word must read 1 here and 0 for the unscaled inputs, and both results must
    match the oracle.  Dense attention runs on the same kernel with each row's first 64-key block's
    maximum fixed: the same guard, the same re-run (the x16 rows exceed that maximum by far more than
    2^64 allows, the plain rows by at most 2^17)."""
    w = synth.WORKLOADS["padded_7x15x16"]
    plain = synth.make_inputs(w)
    x = dict(plain)
    for n in ("q", "k"):
        x[n] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(x[n]) * 16.0)
    s = _shape(w)
    _, C = vsa.shape_info(s)
    k = C if dense else w.topk
    scale = 1 / math.sqrt(w.head_dim)
    ws = vsa.alloc_workspace(s, k)
    for inputs, scaled in ((x, True), (plain, False)):
        f64 = {n: O.bf16_to_f64(v) for n, v in inputs.items()}
        dev = {n: to_dev(v) for n, v in inputs.items()}
        got = from_dev(vsa.forward(dev["q"], dev["k"], dev["v"], s, k, scale, None if dense else dev["g_coarse"],
                                   None if dense else dev["g_fine"], workspace=ws))
        rerun = vsa.forward_rerun(s, k, ws, has_g_coarse=not dense)
        assert np.isfinite(got).all()
        if dense:
            ref, lse = O.dense(f64["q"], f64["k"], f64["v"], w.grid, scale)
            assert (lse.max() > 100) == scaled
            assert rerun == scaled, f"dense overflow re-run {'missing' if scaled else 'fired'}"
        else:
            ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, k, scale, f64["g_coarse"], f64["g_fine"])
            ref = ora["out"]
            assert rerun == scaled, f"overflow re-run {'missing' if scaled else 'fired'} (scaled inputs: {scaled})"
        for b in range(w.batch):
            for h in range(w.heads):
                check_close(got[b, :, h], ref[b, :, h], f"forward(scaled={scaled})[b={b},h={h}]")
    vsa.device_status()


def test_overflow_word_of_the_fused_fine_call():
    """vsa_fine_fused with precomputed steps reports its overflow in the caller's word: 1 on the x16
    inputs (and the re-run's result matches the oracle), 0 on the plain inputs; a stale 1 left in
    the word is cleared by the next call.  The second word is the kernel's work counter: every item
    past the first one of each CTA is claimed from it exactly once, so it ends at the item count."""
    w = synth.WORKLOADS["padded_7x15x16"]
    plain = synth.make_inputs(w)
    scaled = dict(plain)
    for n in ("q", "k"):
        scaled[n] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(scaled[n]) * 16.0)
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    word = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    for inputs, expect in ((scaled, 1), (plain, 0), (scaled, 1)):
        f64 = {n: O.bf16_to_f64(v) for n, v in inputs.items()}
        dev = {n: to_dev(v) for n, v in inputs.items()}
        ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, scale)
        idx = torch.from_numpy(ora["idx"]).cuda()
        got = from_dev(vsa.fine_fused(dev["q"], dev["k"], dev["v"], s, idx, scale, steps=vsa.schedule(idx, s),
                                      overflow=word))
        assert int(word[0].item()) == expect
        _, C = vsa.shape_info(s)
        assert int(word[1].item()) == w.batch * w.heads * ((C + 1) // 2)
        ref = O.untile(ora["o_fine"], w.grid)
        for b in range(w.batch):
            for h in range(w.heads):
                check_close(got[b, :, h], ref[b, :, h], f"fine_fused(expect overflow {expect})[b={b},h={h}]")


def test_padded_key_rows_are_masked():
    """Large finite values written into the padded rows of the tiled K do not change the result."""
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    qt, kt, vt, s = _run_fine(w, x)
    o1, l1 = vsa.fine(qt, kt, vt, s, None)
    pad = torch.from_numpy(~O.key_valid_mask(w.grid)).cuda()
    kt2 = kt.clone()
    kt2[:, :, pad, :] = 1.0e4
    o2, l2 = vsa.fine(qt, kt2, vt, s, None)
    valid = torch.from_numpy(O.key_valid_mask(w.grid)).cuda()
    assert torch.equal(o1[:, :, valid], o2[:, :, valid])
    assert torch.equal(l1[:, :, valid], l2[:, :, valid])


def test_duplicate_and_out_of_range_indices():
    """A listed-twice cube is attended twice; an out-of-range entry is an empty cube."""
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    f64 = {k: O.bf16_to_f64(v) for k, v in x.items()}
    qt, kt, vt, s = _run_fine(w, x)
    npad, C = vsa.shape_info(s)
    rng = np.random.default_rng(3)
    idx = np.sort(rng.integers(0, C, size=(1, w.heads, C, 6)), axis=-1).astype(np.int32)
    idx[..., 1] = idx[..., 0]                      # a duplicate in every row
    bad = idx.copy()
    bad[..., -1] = C + 7                           # and an out-of-range entry
    tq = [O.tile(f64[n], w.grid) for n in ("q", "k", "v")]
    o, lse = vsa.fine(qt, kt, vt, s, torch.from_numpy(idx).cuda())
    r_o, r_lse = O.fine(*tq, idx, 1 / math.sqrt(128), w.grid)
    check_heads(from_dev(o), r_o, w.grid, "o_fine(dup)")
    o2, _ = vsa.fine(qt, kt, vt, s, torch.from_numpy(bad).cuda())
    r_o2, _ = O.fine(*tq, bad[..., :-1], 1 / math.sqrt(128), w.grid)
    check_heads(from_dev(o2), r_o2, w.grid, "o_fine(out of range)")


def test_k_equals_one_and_k_equals_c():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    f64 = {k: O.bf16_to_f64(v) for k, v in x.items()}
    d = {k: to_dev(v) for k, v in x.items()}
    npad, C = vsa.shape_info(_shape(w))
    for k in (1, C):
        _compare_call(w, d, f64, k, 1 / math.sqrt(128))


def test_repeated_calls_are_deterministic():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    s = _shape(w)
    a = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, None, d["g_coarse"], d["g_fine"])
    b = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, None, d["g_coarse"], d["g_fine"])
    assert torch.equal(a, b)


def test_one_tile_kernel_with_many_items_per_cta():
    """160 heads of an 8x8x8 grid at top-k 2: 640 work items of one or two steps over at most one CTA per
    SM, so every CTA carries several items and the per-item hand-overs between the softmax groups, the
    epilogue warps and the next item's first steps happen many times.  The fused fine stage with
    precomputed steps (the one-tile kernel) must match the oracle on every head and give the same bits
    on every one of 20 repeated launches; the whole forward call must repeat bit for bit too, and so
    must dense attention on the same kernel."""
    w = synth.custom_workload("many_items_8x8x8", 1, 160, 64, (8, 8, 8), 2, field=True, wid=97)
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    f64 = {k: O.bf16_to_f64(v) for k, v in x.items()}
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, scale, f64["g_coarse"], f64["g_fine"])
    idx = torch.from_numpy(ora["idx"]).cuda()
    steps = vsa.schedule(idx, s)
    first = vsa.fine_fused(d["q"], d["k"], d["v"], s, idx, scale, steps=steps)
    ref = O.untile(ora["o_fine"], w.grid)
    got = from_dev(first)
    for h in range(w.heads):
        check_close(got[0, :, h], ref[0, :, h], f"many items fine_fused h={h}")
    for rep in range(20):
        again = vsa.fine_fused(d["q"], d["k"], d["v"], s, idx, scale, steps=steps)
        assert torch.equal(again.view(torch.int16), first.view(torch.int16)), f"launch {rep} differs"
    a = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, d["g_coarse"], d["g_fine"])
    for rep in range(5):
        b = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, d["g_coarse"], d["g_fine"])
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"forward call {rep} differs"
    # dense attention on the same kernel: 160 heads x 4 items of four 64-token blocks, claimed by the CTAs
    r_dense, _ = O.dense(f64["q"], f64["k"], f64["v"], w.grid, scale)
    dense = vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale)
    got = from_dev(dense)
    for h in range(w.heads):
        check_close(got[0, :, h], r_dense[0, :, h], f"many items dense h={h}")
    for rep in range(10):
        again = vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale)
        assert torch.equal(again.view(torch.int16), dense.view(torch.int16)), f"dense launch {rep} differs"


HOST_CASES = {
    # name: (workload, gates): 4 heads -> four groups of one head; 1 head -> one group (no pipeline);
    # 11 heads -> groups of two heads with a last group of one, no gates; B = 2, d = 64; 40 heads ->
    # groups of 7 7 7 6 6 4 2 1 heads (the shrinking tail)
    "padded_4_heads": ("padded_7x15x16", True),
    "one_head": (("one_head_7x15x16", 1, 1, 128, (7, 15, 16), 8), True),
    "eleven_heads_no_gates": (("eleven_heads_9x6x5", 2, 11, 64, (9, 6, 5), 4), False),
    "forty_heads": (("forty_heads_7x15x16", 1, 40, 64, (7, 15, 16), 8), True),
}


@pytest.mark.parametrize("name", list(HOST_CASES))
def test_forward_host_matches_device_forward(name):
    """vsa_forward_host (head groups, copy streams, gathered gates) gives the bits of vsa_forward, twice in a
    row on the same workspace (the second call's copies must wait for the first call's work)."""
    spec, gates = HOST_CASES[name]
    w = synth.WORKLOADS[spec] if isinstance(spec, str) else synth.custom_workload(*spec[:5], spec[5], wid=98)
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    h = {k: d[k].cpu().pin_memory() for k in d}
    s = _shape(w)
    gc, gf = (d["g_coarse"], d["g_fine"]) if gates else (None, None)
    hgc, hgf = (h["g_coarse"], h["g_fine"]) if gates else (None, None)
    ref = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, None, gc, gf)
    ws = vsa.alloc_workspace(s, w.topk, host_io=True)
    out1 = torch.empty_like(h["q"]).pin_memory()
    out2 = torch.empty_like(h["q"]).pin_memory()
    vsa.forward_host(h["q"], h["k"], h["v"], s, w.topk, ws, out1, None, hgc, hgf)
    vsa.forward_host(h["q"], h["k"], h["v"], s, w.topk, ws, out2, None, hgc, hgf)
    torch.cuda.current_stream().synchronize()
    r = ref.cpu()
    assert torch.equal(out1, r)
    assert torch.equal(out2, r)


def test_group_is_a_permutation_and_does_not_change_the_output(case):
    """vsa_group only reorders the work.  Any order gives a valid result: the
    fine kernel pairs a row's key cubes into 128-key steps as the group's
    union dictates, which changes only the rounding order, so each order is
    compared with the oracle (its own selection) within the usual tolerances."""
    w, _, dev, f64 = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    qt, kt, vt = (vsa.tile(dev[n], s) for n in ("q", "k", "v"))
    bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
    scores, _ = vsa.coarse(*bars, s, scale)
    order = vsa.group(scores, s)
    _, C = vsa.shape_info(s)
    o = order.cpu().numpy()
    assert np.array_equal(np.sort(o, axis=-1), np.broadcast_to(np.arange(C, dtype=np.int32), o.shape))
    ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, scale)
    idx = torch.from_numpy(ora["idx"]).cuda()
    rev = torch.flip(order, dims=[-1]).contiguous()
    shuffled = torch.from_numpy(np.random.default_rng(0).permuted(
        np.broadcast_to(np.arange(C, dtype=np.int32), o.shape), axis=-1).copy()).cuda()
    valid = O.key_valid_mask(w.grid)
    for name, ordr in (("identity", None), ("group", order), ("reversed", rev), ("shuffled", shuffled)):
        of, lse = vsa.fine(qt, kt, vt, s, idx, scale, order=ordr)
        check_heads(from_dev(of), ora["o_fine"], w.grid, f"o_fine[{name}]")
        assert np.abs(from_dev(lse)[:, :, valid] - ora["lse"][:, :, valid]).max() <= LSE_ABS, name
    r_d, r_dl = O.fine(*(O.tile(f64[n], w.grid) for n in ("q", "k", "v")), None, scale, w.grid)
    for ordr in (None, shuffled):
        d1, dl1 = vsa.fine(qt, kt, vt, s, None, scale, order=ordr)
        check_heads(from_dev(d1), r_d, w.grid, "dense")
        assert np.abs(from_dev(dl1)[:, :, valid] - r_dl[:, :, valid]).max() <= LSE_ABS
    # dense attention walks every cube in the same pairs whatever the order: bit-identical
    d1, _ = vsa.fine(qt, kt, vt, s, None, scale)
    d2, _ = vsa.fine(qt, kt, vt, s, None, scale, order=shuffled)
    assert torch.equal(d1, d2)


def test_group_keys_follow_top_scores():
    """On hand-made scores the order is the sort by each row's top-3 key cubes."""
    w = synth.custom_workload("group_8", 1, 1, 128, (8, 8, 8), 2)
    s = _shape(w)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(4)
    sc = rng.standard_normal((1, 1, C, C)).astype(np.float32)
    top = np.argsort(-sc[0, 0], axis=-1, kind="stable")[:, :3]
    expect = sorted(range(C), key=lambda i: (top[i, 0], top[i, 1], top[i, 2], i))
    got = vsa.group(torch.from_numpy(sc).cuda(), s).cpu().numpy()[0, 0]
    assert got.tolist() == expect


# ---------------------------------------------------------------- fused pipeline entry points
def test_pool_qkv_bit_identical_to_pool_of_tiles(case):
    """Pooling straight from the token layout sums in the same order as pooling the tiled copy."""
    w, _, dev, _ = case
    s = _shape(w)
    bars = vsa.pool_qkv(dev["q"], dev["k"], dev["v"], s)
    for name, got in zip(("q", "k", "v"), bars):
        assert torch.equal(got, vsa.pool(vsa.tile(dev[name], s), s)), name


def test_fine_fused_sparse_matches_oracle(case):
    """Cube gathers from the token layout + merge in the epilogue, on the oracle's selection."""
    w, _, dev, f64 = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    ora = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, scale, f64["g_coarse"], f64["g_fine"])
    idx = torch.from_numpy(ora["idx"]).cuda()
    # fine output alone (no coarse term, g_fine = 1), written in token layout, with the kernel's
    # own walk and with precomputed steps
    ref = O.untile(ora["o_fine"], w.grid)
    for steps in (None, vsa.schedule(idx, s)):
        got = from_dev(vsa.fine_fused(dev["q"], dev["k"], dev["v"], s, idx, scale, steps=steps))
        for b in range(w.batch):
            for h in range(w.heads):
                check_close(got[b, :, h], ref[b, :, h], f"fine_fused[b={b},h={h}] steps={steps is not None}")
    # with the oracle's coarse output and both gates: the whole merged result
    oc = torch.from_numpy(ora["o_coarse"].astype(np.float32)).cuda()
    got = from_dev(vsa.fine_fused(dev["q"], dev["k"], dev["v"], s, idx, scale, None, oc, dev["g_coarse"],
                                  dev["g_fine"]))
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(got[b, :, h], ora["out"][b, :, h], f"fine_fused merged[b={b},h={h}]")


def test_fine_fused_dense_matches_oracle(case):
    """Dense attention over blocks of 64 consecutive real tokens (a ragged last block)."""
    w, _, dev, f64 = case
    s = _shape(w)
    r_out, _ = O.dense(f64["q"], f64["k"], f64["v"], w.grid)
    got = from_dev(vsa.fine_fused(dev["q"], dev["k"], dev["v"], s, None))
    for b in range(w.batch):
        for h in range(w.heads):
            check_close(got[b, :, h], r_out[b, :, h], f"dense fused[b={b},h={h}]")


def test_fine_fused_writes_only_real_tokens_and_ignores_order_for_dense():
    w = synth.WORKLOADS["padded_7x15x16"]
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    s = _shape(w)
    sentinel = torch.full_like(d["q"], float("nan"))
    out = vsa.fine_fused(d["q"], d["k"], d["v"], s, None, out=sentinel.clone())
    assert not torch.isnan(out).any()          # every real token's row was written
    npad, C = vsa.shape_info(s)
    rev = torch.arange(C - 1, -1, -1, dtype=torch.int32, device="cuda").expand(w.batch, w.heads, C).contiguous()
    out2 = vsa.fine_fused(d["q"], d["k"], d["v"], s, None, order=rev)
    assert torch.equal(out, out2)


def test_topk_order_selection_and_order(case):
    """The one-pass selection is exactly vsa_topk's; its work order sorts each head's query cubes by
    their four smallest selected key cubes, then by the cube's own index (checked on the host)."""
    w, _, dev, _ = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    scores, _ = vsa.coarse(*vsa.pool_qkv(dev["q"], dev["k"], dev["v"], s), s, scale)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(2)
    tied = torch.from_numpy(rng.integers(-2, 3, size=(w.batch, w.heads, C, C)).astype(np.float32)).cuda()
    for sc in (scores, tied):
        for k in sorted({1, w.topk, C}):
            idx, order = vsa.topk_order(sc, s, k)
            assert torch.equal(idx, vsa.topk(sc, s, k)), k
            ix = idx.cpu().numpy().reshape(-1, C, k)
            o = order.cpu().numpy().reshape(-1, C)
            for bh in range(ix.shape[0]):
                want = sorted(range(C), key=lambda c: tuple(ix[bh, c, :4].tolist()) + (c,))
                assert o[bh].tolist() == want, (k, bh)


def _scores_f64(qb: np.ndarray, kb: np.ndarray, scale: float) -> np.ndarray:
    """Exact-enough reference: the float32 inputs' dot products in float64, scaled."""
    return scale * np.matmul(qb.astype(np.float64), np.swapaxes(kb.astype(np.float64), -1, -2))


@pytest.mark.parametrize("B,H,D,grid", [(1, 3, 128, (8, 16, 16)), (2, 2, 64, (9, 6, 5)), (1, 2, 128, (21, 30, 52)),
                                        (1, 1, 128, (3, 2, 4)), (1, 2, 64, (24, 32, 28)), (1, 2, 128, (20, 28, 36)),
                                        (2, 1, 64, (5, 9, 9))],
                         ids=["C32", "B2_d64_C12", "C624", "C1", "d64_C336", "C315", "B2_d64_C18"])
def test_coarse_scores_exact_on_small_integers(B, H, D, grid):
    """Pooled vectors of small integers: every bf16 part but the first is zero and every dot product is
    an integer below 2^24, so the split tensor-core product must equal the exact scores bit for bit (a
    check of the operand layout, the parts, the six partial products and the row/column tails).  C a
    multiple of 4 takes the copy-engine paths (scores stored and read back by TMA), C = 1, 315 and 18
    the per-thread loads and stores."""
    s = vsa.Shape(B, H, D, grid)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(C + D)
    q, k = (rng.integers(-8, 9, size=(B, H, C, D)).astype(np.float32) for _ in range(2))
    v = rng.standard_normal((B, H, C, D)).astype(np.float32)
    scores, oc = vsa.coarse(*(torch.from_numpy(x).cuda() for x in (q, k, v)), s, 0.125)
    ref = _scores_f64(q, k, 0.125)
    assert np.array_equal(from_dev(scores), ref)
    r_oc = np.matmul(O.softmax_rows(ref), v.astype(np.float64))
    assert np.linalg.norm(from_dev(oc) - r_oc) / np.linalg.norm(r_oc) <= COARSE_REL_L2


@pytest.mark.parametrize("grid", [(12, 16, 20), (20, 28, 36)], ids=["C60", "C315"])
@pytest.mark.parametrize("D", [64, 128])
def test_coarse_scores_carry_float32_accuracy(D, grid):
    """General float32 pooled vectors (three non-zero parts each) across several magnitudes: every score
    within 2^-19 of the sum of |q_d k_d| from its float64 value (the float32 accumulation of D products
    alone reaches about 2^-20 of it; a dropped or mis-split middle part would miss by about 2^-9 /
    sqrt(D)), and the coarse output within the oracle tolerance."""
    s = vsa.Shape(1, 4, D, grid)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(D + C)
    mag = np.exp(rng.uniform(-6, 6, size=(1, 4, C, 1))).astype(np.float32)
    q = (rng.standard_normal((1, 4, C, D)) * mag).astype(np.float32)
    k = (rng.standard_normal((1, 4, C, D)) * np.exp(rng.uniform(-3, 3, size=(1, 4, C, 1)))).astype(np.float32)
    v = rng.standard_normal((1, 4, C, D)).astype(np.float32)
    scale = 1 / math.sqrt(D)
    scores, oc = vsa.coarse(*(torch.from_numpy(x).cuda() for x in (q, k, v)), s, scale)
    ref = _scores_f64(q, k, scale)
    bound = scale * np.matmul(np.abs(q.astype(np.float64)), np.swapaxes(np.abs(k.astype(np.float64)), -1, -2))
    err = np.abs(from_dev(scores) - ref)
    assert np.all(err <= 2.0 ** -19 * bound), float((err / bound).max())
    r_oc = np.matmul(O.softmax_rows(ref), v.astype(np.float64))
    assert np.linalg.norm(from_dev(oc) - r_oc) / np.linalg.norm(r_oc) <= COARSE_REL_L2


@pytest.mark.parametrize("C_grid", [(24, 32, 52), (20, 32, 44)], ids=["C624", "C440"])
def test_topk_every_search_path(C_grid):
    """The selection on score rows of 440 and 624 cubes, random and tie-heavy, for k on each path of its
    search (one or up to four keys per lane bounding the k-th largest, a compacted list of up to 128 or
    256 candidates, the whole row): bit-exact against the oracle's top-k."""
    s = vsa.Shape(1, 2, 64, C_grid)
    _, C = vsa.shape_info(s)
    rng = np.random.default_rng(C)
    shape = (1, 2, C, C)
    arrays = [rng.standard_normal(shape).astype(np.float32), rng.integers(-3, 4, size=shape).astype(np.float32),
              np.sort(rng.standard_normal(shape).astype(np.float32), axis=-1)]
    for a in arrays:
        dev_a = torch.from_numpy(a).cuda()
        for k in (1, 2, 31, 32, 33, 64, 65, 97, 128, 129, 300, C - 1, C):
            idx, order = vsa.topk_order(dev_a, s, k)
            assert np.array_equal(idx.cpu().numpy(), O.topk(a.astype(np.float64), k)), k
            assert torch.equal(idx, vsa.topk(dev_a, s, k)), k


def _decode_steps(raw: np.ndarray, items: int, stride: int):
    e = raw.view(np.uint32).reshape(items, stride, 2)
    a, b = (e[..., 0] & 0xFFFF).astype(np.int64), (e[..., 0] >> 16).astype(np.int64)
    return a, b, (e[..., 1] & 0xFF).astype(np.int64), (e[..., 1] >> 31).astype(np.int64)


def test_schedule_covers_every_selection_once(case):
    """Bit-exact check of the precomputed steps: each item (a pair of query cubes) visits every
    (query cube, selected key cube) entry of its two lists exactly as often as the lists hold it,
    two key cubes at most per step, in ascending cube order, and the last flag only on the final
    step."""
    w, _, dev, _ = case
    s = _shape(w)
    scale = 1 / math.sqrt(w.head_dim)
    scores, _ = vsa.coarse(*vsa.pool_qkv(dev["q"], dev["k"], dev["v"], s), s, scale)
    _, C = vsa.shape_info(s)
    k = w.topk
    idx, order = vsa.topk_order(scores, s, k)
    rng = np.random.default_rng(9)
    dup = idx.cpu().numpy().copy()
    if k >= 2:
        dup[..., 1] = dup[..., 0]                       # duplicates must be visited twice
    dup[..., -1] = np.where(rng.random(dup.shape[:-1]) < 0.2, C + 3, dup[..., -1])   # out of range: empty cube
    for sel in (idx.cpu().numpy(), dup):
        steps = vsa.schedule(torch.from_numpy(sel).cuda(), s, order).cpu().numpy()
        groups = (C + 1) // 2   # a work item is a pair of query cubes (one 128-row tile)
        items, stride = w.batch * w.heads * groups, k
        a, b, fl, last = _decode_steps(steps, items, stride)
        o = order.cpu().numpy().reshape(-1, C)
        for it in range(items):
            bh, g = divmod(it, groups)
            cubes = [o[bh, 2 * g + j] if 2 * g + j < C else -1 for j in range(2)]
            want = {}
            for j, c in enumerate(cubes):
                if c < 0:
                    continue
                for kc in sel.reshape(-1, C, k)[bh, c]:
                    key = (j, int(kc) if 0 <= kc < C else C)
                    want[key] = want.get(key, 0) + 1
            got, pats = {}, []
            n = int(np.argmax(last[it] == 1)) + 1
            assert last[it, :n].sum() == 1
            for st in range(n):
                for blk, f in ((a[it, st], fl[it, st] & 15), (b[it, st], fl[it, st] >> 4)):
                    if blk == 0xFFFF:
                        assert f == 0
                        continue
                    pats.append(((1 if f & 3 else 0) | (2 if f & 12 else 0), int(blk)))
                    for j in range(4):
                        if f >> j & 1:
                            got[(j, int(blk))] = got.get((j, int(blk)), 0) + 1
            assert got == want, it
            assert pats == sorted(pats), it
