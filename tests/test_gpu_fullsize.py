"""Parity at the full Wan 480p / 720p sizes, in the launch configuration the
benchmark times (the whole call on one stream), checked on sampled heads and
query cubes that the oracle computes one by one, plus properties that hold at
any size (tile round trip, whole call == the per-step path up to rounding)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cube_b200 as vsa
import synth
from oracle import vsa_oracle as O
from tests._util import (COARSE_REL_L2, LSE_ABS, assert_selection, bf16_bits, check_close, from_dev, to_dev)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["wan480p_dense", "wan480p_vsa_k32", "wan720p_cfg_k64"]


@pytest.fixture(scope="module", params=FULL)
def run(request):
    w = synth.WORKLOADS[request.param]
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    npad, C = vsa.shape_info(s)
    scale = 1 / math.sqrt(w.head_dim)
    dense = w.topk == C
    r = {"w": w, "x": x, "s": s, "C": C, "scale": scale, "dense": dense}
    gc, gf = (None, None) if dense else (d["g_coarse"], d["g_fine"])
    r["out"] = vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, gc, gf)
    qt, kt, vt = (vsa.tile(d[n], s) for n in ("q", "k", "v"))
    r["rt_ok"] = all(torch.equal(vsa.untile(t, s), d[n]) for t, n in ((qt, "q"), (kt, "k"), (vt, "v")))
    if dense:
        o, lse = vsa.fine(qt, kt, vt, s, None, scale)
        stage_out = vsa.untile(o, s)
    else:
        bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
        scores, oc = vsa.coarse(*bars, s, scale)
        idx = vsa.topk(scores, s, w.topk)
        o, lse = vsa.fine(qt, kt, vt, s, idx, scale, order=vsa.group(scores, s))
        stage_out = vsa.untile(vsa.combine(oc, o, s, gc, gf), s)
        r["bars"] = [b.cpu() for b in bars]
        r["scores"] = scores.cpu()
        r["oc"] = oc.cpu()
        r["idx"] = idx.cpu().numpy()
    fused, staged = r["out"].float(), stage_out.float()
    if dense:
        # different block order (64 consecutive real tokens instead of cubes): a different
        # but equally valid rounding order, so the oracle tolerance applies
        err = fused - staged
        r["stage_close"] = bool(err.abs().max() <= 2e-2) and bool(err.norm() <= 5e-3 * staged.norm())
    else:
        # identical selections; the forward call's steps come in another (precomputed) order,
        # so the oracle tolerance applies, per head
        err = (fused - staged).float()
        ok = True
        for b in range(fused.shape[0]):
            for h in range(fused.shape[2]):
                e, ref = err[b, :, h], staged[b, :, h]
                ok = ok and bool(e.abs().max() <= 2e-2) and bool(e.norm() <= 5e-3 * ref.norm())
        r["stage_close"] = ok
    r["qt_rows"] = qt
    r["o_fine"] = o.cpu()
    r["lse"] = lse.cpu()
    r["out"] = r["out"].cpu()
    torch.cuda.synchronize()
    del qt, kt, vt, d
    torch.cuda.empty_cache()
    return r


def _sample_heads(w):
    hs = sorted({0, w.heads // 2, w.heads - 1})
    return [(b, h) for b in range(w.batch) for h in hs]


def _sample_cubes(C, n=12, seed=0):
    rng = np.random.default_rng(seed)
    return sorted({0, C - 1, C // 2} | set(rng.integers(0, C, size=n).tolist()))


def test_roundtrip_and_stage_equivalence(run):
    assert run["rt_ok"]
    assert run["stage_close"], "vsa_forward differs from the per-step path beyond rounding"


def test_tile_sampled_rows(run):
    w, x = run["w"], run["x"]
    src = O.tile_source_index(w.grid)
    rng = np.random.default_rng(1)
    qt = run["qt_rows"]
    npad = src.size
    for b, h in _sample_heads(w):
        ps = rng.integers(0, npad, size=256)
        got = bf16_bits(qt[b, h, torch.from_numpy(ps).cuda()])
        for i, p in enumerate(ps):
            exp = x["q"][b, src[p], h] if src[p] >= 0 else np.zeros(w.head_dim, np.uint16)
            assert np.array_equal(got[i], exp), (b, h, p)


def _head_f64(x, b, h, name, grid):
    return O.tile(O.bf16_to_f64(x[name][b:b + 1, :, h:h + 1]), grid)[0, 0]


def _oracle_head(run, b, h):
    """Oracle pool, coarse and selection of one head, from the inputs alone."""
    w, x = run["w"], run["x"]
    tiled = [_head_f64(x, b, h, n, w.grid) for n in ("q", "k", "v")]
    bars = [O.pool(t[None, None], w.grid)[0, 0] for t in tiled]
    scores, oc = O.coarse(*bars, run["scale"])
    return tiled, bars, scores, oc, O.topk(scores, w.topk)


def test_selection_sampled_heads(run):
    if run["dense"]:
        pytest.skip("dense call has no selection")
    w, k = run["w"], run["w"].topk
    for b, h in _sample_heads(w):
        _, r_bars, r_scores, r_oc, r_idx = _oracle_head(run, b, h)
        for bar, r in zip(run["bars"], r_bars):
            np.testing.assert_allclose(bar[b, h].numpy().astype(np.float64), r, rtol=1e-5, atol=1e-6)
        g_scores = run["scores"][b, h].numpy().astype(np.float64)
        np.testing.assert_allclose(g_scores, r_scores, rtol=0, atol=1e-5 * np.abs(r_scores).max())
        g_oc = run["oc"][b, h].numpy().astype(np.float64)
        assert np.linalg.norm(g_oc - r_oc) / np.linalg.norm(r_oc) <= COARSE_REL_L2
        assert_selection(run["idx"][b, h], r_idx, r_scores, k, f"{w.name} b={b} h={h}")


def test_fine_and_output_sampled_cubes(run):
    """Sampled query cubes against the oracle's fine step and merge.  The oracle runs each cube
    over the GPU's own selection, so a documented near-tie swap (checked and counted by
    test_selection_sampled_heads) is compared like any other cube instead of being left out."""
    w, x, C = run["w"], run["x"], run["C"]
    kv = O.key_valid_mask(w.grid)
    src = O.tile_source_index(w.grid)
    compared = swapped = 0
    for b, h in _sample_heads(w):
        if run["dense"]:
            qt, kt, vt = (_head_f64(x, b, h, n, w.grid) for n in ("q", "k", "v"))
        else:
            (qt, kt, vt), _, _, r_oc, r_idx = _oracle_head(run, b, h)
        for i in _sample_cubes(C, n=6 if run["dense"] else 12, seed=b * 1000 + h):
            if run["dense"]:
                sel = range(C)
            else:
                sel = run["idx"][b, h, i]
                swapped += int(not np.array_equal(sel, r_idx[i]))
            r = slice(i * 64, (i + 1) * 64)
            ro, rl = O.fine_cube(qt[r], kt, vt, sel, kv, run["scale"])
            valid = kv[r]
            got = from_dev(run["o_fine"][b, h, r])
            check_close(got[valid], ro[valid], f"o_fine b={b} h={h} cube={i}")
            lse = run["lse"][b, h, r].numpy().astype(np.float64)
            assert np.abs(lse[valid] - rl[valid]).max() <= LSE_ABS, (b, h, i)
            toks = src[r][valid]
            if run["dense"]:
                ref_out = ro[valid]
            else:
                gc = O.bf16_to_f64(x["g_coarse"][b, toks, h])[:, None]
                gf = O.bf16_to_f64(x["g_fine"][b, toks, h])[:, None]
                ref_out = gc * r_oc[i][None, :] + gf * ro[valid]
            got_out = O.bf16_to_f64(bf16_bits(run["out"][b, torch.from_numpy(toks), h]))
            check_close(got_out, ref_out, f"out b={b} h={h} cube={i}")
            compared += 1
    assert swapped <= max(1, 0.02 * compared), f"{swapped} of {compared} sampled cubes carry a near-tie swap"
    print(f"{w.name}: {compared} sampled query cubes compared, {swapped} with a near-tie swap")
