"""Run the stages of one attention call on a named synthetic workload and print their times.

    python -m block_sparse_attention_cube_b200.run_case --workload wan480p_vsa_k32 --iters 3

Each iteration runs the launches of vsa_forward one by one through the C ABI,
pool_qkv -> coarse -> topk_order -> schedule -> fine_fused (fine_fused alone, dense,
when top-k covers every cube), with CUDA events between the stages.
`--dense-too` adds a dense fine_fused launch on the same inputs.  `--staged`
runs the unfused per-step path instead (tile -> pool -> coarse -> top-k ->
group -> fine -> combine -> untile).  Useful on its own and as a small, fixed
case to put under a profiler.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

import block_sparse_attention_cube_b200 as vsa  # noqa: E402


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="wan480p_vsa_k32", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--dense-too", action="store_true")
    ap.add_argument("--staged", action="store_true")
    a = ap.parse_args(argv)
    w = synth.WORKLOADS[a.workload]
    x = synth.make_inputs(w)
    d = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in x.items()}
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    npad, C = vsa.shape_info(s)
    scale = 1.0 / math.sqrt(w.head_dim)
    dense = w.topk == C
    if a.staged:
        names = ["tile", "fine", "untile"] if dense else ["tile", "pool", "coarse", "topk+group", "fine", "combine",
                                                           "untile"]
    else:
        names = ["fine"] if dense else ["pool", "coarse", "topk_order", "schedule", "fine"]
    if a.dense_too:
        names.append("fine_dense")
    times = {n: [] for n in names}
    stream = torch.cuda.current_stream()
    for _ in range(a.iters):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        i = 0

        def mark():
            nonlocal i
            ev[i].record(stream)
            i += 1

        mark()
        if a.staged:
            qt, kt, vt = (vsa.tile(d[n], s) for n in ("q", "k", "v"))
            mark()
            if dense:
                of, _ = vsa.fine(qt, kt, vt, s, None, scale, want_lse=False)
                mark()
                vsa.untile(of, s)
                mark()
            else:
                bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
                mark()
                scores, oc = vsa.coarse(*bars, s, scale)
                mark()
                idx = vsa.topk(scores, s, w.topk)
                order = vsa.group(scores, s)
                mark()
                of, _ = vsa.fine(qt, kt, vt, s, idx, scale, want_lse=False, order=order)
                mark()
                ot = vsa.combine(oc, of, s, d["g_coarse"], d["g_fine"])
                mark()
                vsa.untile(ot, s)
                mark()
            if a.dense_too:
                vsa.fine(qt, kt, vt, s, None, scale, want_lse=False)
                mark()
        else:
            if dense:
                vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale)
                mark()
            else:
                bars = vsa.pool_qkv(d["q"], d["k"], d["v"], s)
                mark()
                scores, oc = vsa.coarse(*bars, s, scale)
                mark()
                idx, order = vsa.topk_order(scores, s, w.topk)
                mark()
                steps = vsa.schedule(idx, s, order)
                mark()
                vsa.fine_fused(d["q"], d["k"], d["v"], s, idx, scale, order, oc, d["g_coarse"], d["g_fine"],
                               steps=steps)
                mark()
            if a.dense_too:
                vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale)
                mark()
        torch.cuda.synchronize()
        for j, n in enumerate(names):
            times[n].append(ev[j].elapsed_time(ev[j + 1]))
    vsa.device_status()
    print(json.dumps({"workload": w.name, "iters": a.iters,
                      "ms": {n: round(statistics.median(v), 4) for n, v in times.items()}}))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
