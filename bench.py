"""Benchmark of the B200 VSA / dense attention path at the Wan 480p workload.

One step = one VSA call (grid 21x30x52 -> 39,936 padded tokens, 624 cubes,
40 heads, d=128, top-k 32 cubes, gated coarse + fine output) and one dense
attention call on the same Q/K/V (every cube selected, no gates), both
through the library's C ABI on one stream with inputs resident in HBM; the
timed region runs the K steps' dense calls back to back, then their VSA
calls (the two kinds alternating are reported on their own afterwards).

Prints one JSON line.  `value` is the median milliseconds per VSA call (whole
job: with N GPUs, N independent calls complete per step, so value = step
time / N for the VSA part); the dense call is reported beside it.  Timing:
CUDA events on the launching stream after warm-up, synchronize + barrier
around the timed region, max over ranks, medians over the timed calls.
Inputs (1.0 GB of Q/K/V per call) exceed the 126 MB L2, so L2 is not flushed
between steps.  After the timed region, on the same process: the per-stage
breakdown of the call, the Wan 720p CFG batch (2 x 21x45x80 tokens, top-k
64), the memory-bound entry points one by one (HBM GB/s), the pre-attention
pass, the end-to-end call on host buffers, and (rank 0, one GPU) the oracle
on the host cores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --stages [--workload NAME] [--iters I] [--dense-too] [--staged]
    python bench.py --calls [--workload NAME] [--iters I]

`--impl reference` times the fp64 CPU oracle, one whole head per step, on
rank 0 only.  `--stages` runs the launches of one call stage by stage on a
named workload and prints their median times, and `--calls` runs whole
forward calls on it (small fixed cases to put under a profiler).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "ms per VSA/dense attention call at 480p (40 heads, d=128); fine-kernel % BF16 peak"
WORKLOAD = "wan480p_vsa_k32"
DENSE_WORKLOAD = "wan480p_dense"
CFG_WORKLOAD = "wan720p_cfg_k64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# oracle sample: step s runs the whole call (tile .. untile) on head (ORACLE_STRIDE * s) mod H
# of batch element 0; the per-call figure is the median head time times B * H
ORACLE_STRIDE = 7
ORACLE_BASELINE_HEADS = 12


# ---------------------------------------------------------------- shared helpers
def executed_fine_flops(batch: int, heads: int, npad: int, k: int, d: int) -> float:
    """QK^T and PV over 64x64 cube tiles for the k selected cubes of every query cube."""
    return 4.0 * batch * heads * npad * k * 64 * d


def dense_equivalent_flops(batch: int, heads: int, n: int, d: int) -> float:
    return 4.0 * batch * heads * n * n * d


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def reduce_max(value: float, world: int) -> float:
    """Max over ranks (identity on one process)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_ms_per_call(max_step_ms: float, calls_per_step_per_rank: int, world: int) -> float:
    """Weak scaling: every rank runs its own calls; the job completes world*calls per step."""
    return max_step_ms / (calls_per_step_per_rank * world)


def memory_bytes(w, npad: int, c: int) -> dict:
    """Algorithmic HBM bytes per launch of the memory-bound entry points (each input read once, each
    output written once; padded rows are neither read nor needed where the kernel skips them)."""
    tok = w.batch * w.tokens * w.heads * w.head_dim * 2          # one [B, N, H, D] bf16 tensor
    til = w.batch * w.heads * npad * w.head_dim * 2             # one [B, H, Npad, D] bf16 tensor
    bar = w.batch * w.heads * c * w.head_dim * 4                # one [B, H, C, D] fp32 tensor
    gate = w.batch * w.tokens * w.heads * 2
    return {
        "tile": tok + til,                                      # real rows read, every row written (zeros)
        "untile": 2 * tok,                                      # real rows read and written
        "pool": tok + bar,                                      # real rows of one tiled tensor read
        "pool_qkv": 3 * (tok + bar),
        "combine": tok + 2 * gate + bar + til,                  # O_f real rows, gates, O_c; every row written
        "topk": w.batch * w.heads * c * c * 4 + w.batch * w.heads * c * w.topk * 4,
    }


def traffic_for(kernel_src: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(kernel_src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    e = rec.get(key)
    if not e or e.get("source_sha256") != sha:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu_id], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        sm, mx, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.read().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) != len(self.FIELDS):
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "power_w_max": max(power),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- the oracle
def oracle_head_seconds(w, x, h: int) -> float:
    """Seconds the fp64 oracle takes for the whole call (tile, pool, coarse, top-k, fine, merge,
    untile) on head h of batch element 0; decoding the bf16 inputs is not timed."""
    from oracle import vsa_oracle as O
    scale = 1.0 / math.sqrt(w.head_dim)
    f = {n: O.bf16_to_f64(x[n][:1, :, h:h + 1]) for n in x}
    t0 = time.perf_counter()
    O.forward(f["q"], f["k"], f["v"], w.grid, w.topk, scale, f["g_coarse"], f["g_fine"])
    return time.perf_counter() - t0


def oracle_sample_heads(w, steps: range):
    return [(ORACLE_STRIDE * s) % w.heads for s in steps]


def oracle_rule_text(w) -> str:
    return (f"{w.name}: whole oracle call (tile, pool, coarse, top-k, fine over all {synth_cubes(w)} query cubes, "
            f"merge, untile) on one head per step, head (7*step) mod {w.heads} of batch element 0; "
            f"per-call figure = median head time x B*H = {w.batch * w.heads} heads")


def synth_cubes(w) -> int:
    return math.prod((a + 3) // 4 for a in w.grid)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, rank: int):
    if rank != 0:
        return
    w = synth.WORKLOADS[WORKLOAD]
    x = synth.make_inputs(w)
    for h in oracle_sample_heads(w, range(args.warmup)):
        oracle_head_seconds(w, x, h)
    secs = []
    t0 = time.perf_counter()
    for h in oracle_sample_heads(w, range(args.warmup, args.warmup + args.steps)):
        secs.append(oracle_head_seconds(w, x, h))
    wall_ms_per_step = (time.perf_counter() - t0) * 1e3 / args.steps
    per_call_ms = statistics.median(secs) * w.batch * w.heads * 1e3
    cores = blas_threads()
    sample = oracle_rule_text(w) + f"; {args.steps} timed steps, {sum(secs):.1f} s of CPU work"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(per_call_ms, 2), "unit": "ms", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall_ms_per_step, 2),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Philox, Wan 480p field inputs)",
        "config": {"workload": WORKLOAD, "batch": w.batch, "grid": "x".join(map(str, w.grid)), "heads": w.heads,
                   "head_dim": w.head_dim, "topk": w.topk},
        "extrapolated": {"ms_per_call": round(per_call_ms, 2), "from": "median head time x B*H",
                         "step": "one whole head of the call per step (ms_per_step is its measured wall time)"},
        "cpu_baseline": {"value": round(per_call_ms, 2), "unit": "ms", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(per_call_ms, 2), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- the CUDA arm
def _events(torch, n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def stage_times(vsa, torch, d, w, iters: int, warmup: int, dense_too: bool = False, staged: bool = False):
    """Median ms of each launch group of one call, run stage by stage through the entry points."""
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    _, C = vsa.shape_info(s)
    scale = 1.0 / math.sqrt(w.head_dim)
    dense = w.topk == C
    stream = torch.cuda.current_stream()
    out = torch.empty_like(d["q"])
    word = torch.zeros(4, dtype=torch.int32, device=d["q"].device)
    acc = {}
    for it in range(warmup + iters):
        marks = []

        def mark(name=None):
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            marks.append((name, e))

        mark()
        if staged:
            qt, kt, vt = (vsa.tile(d[n], s) for n in ("q", "k", "v"))
            mark("tile")
            if dense:
                of, _ = vsa.fine(qt, kt, vt, s, None, scale, want_lse=False)
                mark("fine")
                vsa.untile(of, s)
                mark("untile")
            else:
                bars = [vsa.pool(t, s) for t in (qt, kt, vt)]
                mark("pool")
                scores, oc = vsa.coarse(*bars, s, scale)
                mark("coarse")
                idx = vsa.topk(scores, s, w.topk)
                order = vsa.group(scores, s)
                mark("topk+group")
                of, _ = vsa.fine(qt, kt, vt, s, idx, scale, want_lse=False, order=order)
                mark("fine")
                ot = vsa.combine(oc, of, s, d["g_coarse"], d["g_fine"])
                mark("combine")
                vsa.untile(ot, s)
                mark("untile")
            if dense_too:
                vsa.fine(qt, kt, vt, s, None, scale, want_lse=False)
                mark("fine_dense")
        else:
            if dense:
                vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale, out=out, overflow=word)
                mark("fine")
            else:
                bars = vsa.pool_qkv(d["q"], d["k"], d["v"], s)
                mark("pool")
                scores, oc = vsa.coarse(*bars, s, scale)
                mark("coarse")
                idx, order = vsa.topk_order(scores, s, w.topk)
                mark("topk_order")
                steps = vsa.schedule(idx, s, order)
                mark("schedule")
                vsa.fine_fused(d["q"], d["k"], d["v"], s, idx, scale, order, oc, d["g_coarse"], d["g_fine"],
                               out=out, steps=steps, overflow=word)
                mark("fine")
            if dense_too:
                vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale, out=out, overflow=word)
                mark("fine_dense")
        torch.cuda.synchronize()
        if it >= warmup:
            for (_, e0), (name, e1) in zip(marks, marks[1:]):
                acc.setdefault(name, []).append(e0.elapsed_time(e1))
    return {n: round(statistics.median(v), 4) for n, v in acc.items()}


def time_launches(torch, fn, iters: int, warmup: int = 3) -> float:
    """Median ms of fn() over `iters` launches, each bracketed by events on the current stream."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    ev = [_events(torch, 2) for _ in range(iters)]
    for e in ev:
        e[0].record(stream)
        fn()
        e[1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(e[0].elapsed_time(e[1]) for e in ev)


def memory_kernels(vsa, torch, d, w, hbm_peak: float, iters: int) -> dict:
    """The memory-bound entry points one launch at a time on the 480p tensors: median ms, GB/s of
    algorithmic bytes, fraction of the measured HBM copy bandwidth."""
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    npad, C = vsa.shape_info(s)
    nbytes = memory_bytes(w, npad, C)
    qt = vsa.tile(d["q"], s)
    back = torch.empty_like(d["q"])
    qbar = vsa.pool(qt, s)
    kbar, vbar = vsa.pool(vsa.tile(d["k"], s), s), vsa.pool(vsa.tile(d["v"], s), s)
    scores, oc = vsa.coarse(qbar, kbar, vbar, s)
    of = qt   # any finite tiled tensor stands in for O_f: the merge's traffic does not depend on values
    fns = {
        "tile": lambda: vsa.tile(d["q"], s, out=qt),
        "untile": lambda: vsa.untile(qt, s, out=back),
        "pool": lambda: vsa.pool(qt, s),
        "pool_qkv": lambda: vsa.pool_qkv(d["q"], d["k"], d["v"], s),
        "combine": lambda: vsa.combine(oc, of, s, d["g_coarse"], d["g_fine"]),
        "topk": lambda: vsa.topk(scores, s, w.topk),
    }
    rec = {}
    for name, fn in fns.items():
        ms = time_launches(torch, fn, iters)
        gbs = nbytes[name] / (ms * 1e-3) / 1e9
        rec[name] = {"ms": round(ms, 4), "bytes": nbytes[name], "gbps": round(gbs, 1),
                     "frac_hbm": round(gbs / hbm_peak, 4)}
    del qt, back, scores
    return rec


def cfg720_record(vsa, torch, dev, bf16_peak: float, iters: int, warmup: int) -> dict:
    """The Wan 720p CFG batch (2 x 21x45x80 tokens, 1,440 cubes, top-k 64) through vsa_forward."""
    w = synth.WORKLOADS[CFG_WORKLOAD]
    x = synth.make_inputs(w)
    d = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in x.items()}
    del x
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    npad, C = vsa.shape_info(s)
    scale = 1.0 / math.sqrt(w.head_dim)
    ws = vsa.alloc_workspace(s, w.topk, device=dev)
    out = torch.empty_like(d["q"])
    ms = time_launches(torch, lambda: vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, d["g_coarse"],
                                                  d["g_fine"], workspace=ws, out=out), iters, warmup)
    stages = stage_times(vsa, torch, d, w, iters, warmup)
    vsa.device_status()
    flops = executed_fine_flops(w.batch, w.heads, npad, w.topk, w.head_dim)
    tf = flops / (stages["fine"] * 1e-3) / 1e12
    del d, ws, out
    torch.cuda.empty_cache()
    return {"workload": CFG_WORKLOAD, "batch": w.batch, "grid": "x".join(map(str, w.grid)), "padded_tokens": npad,
            "cubes": C, "heads": w.heads, "head_dim": w.head_dim, "topk": w.topk,
            "ms_per_call": round(ms, 4), "stage_ms": stages,
            "fine": {"executed_tflop": round(flops / 1e12, 3), "tflops": round(tf, 1),
                     "frac_bf16_peak": round(tf / bf16_peak, 4),
                     "dense_equivalent_tflops": round(dense_equivalent_flops(w.batch, w.heads, w.tokens, w.head_dim)
                                                      / (stages["fine"] * 1e-3) / 1e12, 1)}}


def run_cuda(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import block_sparse_attention_cube_b200 as vsa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    w = synth.WORKLOADS[WORKLOAD]
    wd = synth.WORKLOADS[DENSE_WORKLOAD]
    assert wd.grid == w.grid and wd.data_wid == 0 and w.data_wid == 3   # same Q/K/V
    x = synth.make_inputs(w)
    d = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in x.items()}
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    npad, C = vsa.shape_info(s)
    scale = 1.0 / math.sqrt(w.head_dim)
    ws = vsa.alloc_workspace(s, w.topk, device=dev)
    ws_dense = vsa.alloc_workspace(s, C, device=dev)
    out = torch.empty_like(d["q"])
    out_d = torch.empty_like(d["q"])

    def vsa_call():
        vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, d["g_coarse"], d["g_fine"], workspace=ws, out=out)

    def dense_call():
        vsa.forward(d["q"], d["k"], d["v"], s, C, scale, workspace=ws_dense, out=out_d)

    def block(fn, evs=None):
        # the calls of one kind back to back, each between two events when evs is given
        for i in range(len(evs) if evs is not None else args.warmup):
            if evs is not None:
                evs[i][0].record(stream)
            fn()
            if evs is not None:
                evs[i][1].record(stream)

    # A step is one VSA call and one dense call; the K steps' dense calls run back to back, then their
    # VSA calls (in a DiT every layer's attention is of one kind), so the VSA block starts at the clock
    # the dense block's power draw leaves.  Alternating the two made each call run at the clock the
    # other kind left behind: that is reported separately below.  Each kind's per-stage breakdown
    # follows its own block: the VSA stages right after the timed region, then the dense fine stage.
    block(vsa_call)
    block(dense_call)
    vsa.device_status()
    ev_v = [_events(torch, 2) for _ in range(args.steps)]
    ev_d = [_events(torch, 2) for _ in range(args.steps)]
    t_start, t_end = _events(torch, 2)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    block(dense_call, ev_d)
    block(vsa_call, ev_v)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    vsa.device_status()
    step_ms = t_start.elapsed_time(t_end) / args.steps
    vsa_ms = statistics.median(a.elapsed_time(b) for a, b in ev_v)
    dense_ms = statistics.median(a.elapsed_time(b) for a, b in ev_d)
    step_ms_max = reduce_max(step_ms, world)
    vsa_ms_max = reduce_max(vsa_ms, world)
    dense_ms_max = reduce_max(dense_ms, world)

    rerun = vsa.forward_rerun(s, w.topk, ws, has_g_coarse=True)
    rerun_dense = vsa.forward_rerun(s, C, ws_dense, has_g_coarse=False)

    peaks, peaks_src = load_peaks()
    bf16_peak = float(peaks["bf16_tflops"])
    hbm_peak = float(peaks["hbm_gbs"])

    # ---- per-stage breakdown: the launches of vsa_forward, one by one through the entry points; the VSA
    # calls' stages back to back right after the VSA block, then the dense calls' fine stage
    stage_ms = stage_times(vsa, torch, d, w, args.steps, args.warmup)
    stage_ms["fine_dense"] = stage_times(vsa, torch, d, wd, max(5, args.steps // 5), 3)["fine"]

    # ---- the same calls alternating (after the stage breakdown): each call follows the other kind
    pairs = max(5, args.steps // 5)
    ev_alt = [_events(torch, 3) for _ in range(pairs)]
    for e in ev_alt:
        e[0].record(stream)
        vsa_call()
        e[1].record(stream)
        dense_call()
        e[2].record(stream)
    torch.cuda.synchronize()
    interleaved = {"pairs": pairs,
                   "vsa_ms": round(statistics.median(e[0].elapsed_time(e[1]) for e in ev_alt), 4),
                   "dense_ms": round(statistics.median(e[1].elapsed_time(e[2]) for e in ev_alt), 4),
                   "note": "VSA and dense calls alternating, after the stage breakdown; not part of value"}

    # ---- the memory-bound entry points one launch at a time
    mem = memory_kernels(vsa, torch, d, w, hbm_peak, max(10, args.steps))

    # ---- the pre-attention pass (Q/K RMSNorm + 3D RoPE) on the same Q/K, timed on its own
    wts = synth.make_projection_inputs(synth.custom_workload("weights", 1, w.heads, w.head_dim, (1, 1, 1), 1))
    w_q, w_k = (torch.from_numpy(wts[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("w_q", "w_k"))
    q_n, k_n = torch.empty_like(d["q"]), torch.empty_like(d["k"])
    pre_ms = reduce_max(time_launches(torch, lambda: vsa.qk_norm_rope(d["q"], d["k"], s, w_q, w_k, out=(q_n, k_n)),
                                      max(10, args.steps), args.warmup), world)
    del q_n, k_n

    # ---- end to end through vsa_forward_host (pinned host buffers, copies inside the timed region)
    h = {k: v.cpu().pin_memory() for k, v in d.items()}
    h_out = torch.empty_like(h["q"]).pin_memory()
    ws_host = vsa.alloc_workspace(s, w.topk, host_io=True, device=dev)
    e2e_ms = reduce_max(time_launches(
        torch, lambda: vsa.forward_host(h["q"], h["k"], h["v"], s, w.topk, ws_host, h_out, scale, h["g_coarse"],
                                        h["g_fine"]), max(5, args.steps // 2), max(1, args.warmup // 2)), world)
    vsa.device_status()
    h2d = sum(h[k].numel() * 2 for k in ("q", "k", "v", "g_coarse", "g_fine"))
    d2h = h_out.numel() * 2
    del h, h_out, ws_host, ws, ws_dense, out, out_d, d
    torch.cuda.empty_cache()

    # ---- the 720p CFG batch
    cfg = cfg720_record(vsa, torch, dev, bf16_peak, max(5, args.steps // 2), args.warmup)

    if rank != 0:
        return
    pre_bytes = 4 * w.batch * w.tokens * w.heads * w.head_dim * 2
    fine_flops = executed_fine_flops(w.batch, w.heads, npad, w.topk, w.head_dim)
    nblk = (w.tokens + 63) // 64   # dense attention walks blocks of 64 consecutive real tokens
    dense_flops = dense_equivalent_flops(w.batch, w.heads, 64 * nblk, w.head_dim)
    fine_tflops = fine_flops / (stage_ms["fine"] * 1e-3) / 1e12
    dense_tflops = dense_flops / (stage_ms["fine_dense"] * 1e-3) / 1e12
    fine_src = os.path.join(ROOT, "block_sparse_attention_cube_b200", "csrc", "vsa_fine.cu")
    traffic = traffic_for(fine_src, "fine_kernel_wan480p_vsa_k32")
    cpu = None
    if world == 1:
        heads = oracle_sample_heads(w, range(ORACLE_BASELINE_HEADS))
        secs = [oracle_head_seconds(w, x, hh) for hh in heads]
        cpu = {"value": round(statistics.median(secs) * w.batch * w.heads * 1e3, 1), "unit": "ms",
               "cores": blas_threads(), "kind": "oracle",
               "sample": oracle_rule_text(w) + f"; steps 0..{len(heads) - 1}, heads {heads}, "
                                               f"{sum(secs):.1f} s of CPU work"}
    line = {
        "metric": METRIC, "value": round(whole_job_ms_per_call(vsa_ms_max, 1, world), 4), "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox; Q/K = 0.5 N(0,1) + sin(0.3t+0.2x+0.1y+phi), V ~ N(0,1), gates U(0,1))",
        "config": {"workload": WORKLOAD, "batch": w.batch, "grid": "x".join(map(str, w.grid)),
                   "padded_tokens": npad, "cubes": C, "heads": w.heads, "head_dim": w.head_dim, "topk": w.topk,
                   "dense_call": {"workload": DENSE_WORKLOAD, "topk": C},
                   "l2": "no flush: 1.0 GB of Q/K/V per call exceeds the 126 MB L2",
                   "timing": "median of the timed calls (CUDA events on the launching stream); the K dense "
                             "calls back to back, then the K VSA calls",
                   "parallelism": f"{world} independent replicas (weak scaling)"},
        "dense_ms_per_call": round(whole_job_ms_per_call(dense_ms_max, 1, world), 4),
        "stage_ms": stage_ms,
        "fixed_max_rerun": {"vsa": rerun, "dense": rerun_dense},
        "interleaved": interleaved,
        "fine": {"executed_tflop": round(fine_flops / 1e12, 4), "tflops": round(fine_tflops, 1),
                 "frac_bf16_peak": round(fine_tflops / bf16_peak, 4),
                 "dense_equivalent_tflops": round(dense_equivalent_flops(w.batch, w.heads, w.tokens, w.head_dim)
                                                  / (stage_ms["fine"] * 1e-3) / 1e12, 1)},
        "dense_fine": {"executed_tflop": round(dense_flops / 1e12, 3), "tflops": round(dense_tflops, 1),
                       "frac_bf16_peak": round(dense_tflops / bf16_peak, 4),
                       "kernel": "fine_tile_kernel<128, tokens> (the one-tile kernel over blocks of real tokens)",
                       "traffic": traffic_for(fine_src, "fine_kernel_wan480p_dense"),
                       "per_launch": "4*B*H*(64*ceil(N/64))^2*D: blocks of 64 real tokens, no padding"},
        "roofline": {"kernel": "fine_tile_kernel<128, cubes> (VSA, top-k 32)", "bound": "tensor",
                     "achieved": round(fine_tflops, 2),
                     "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(fine_tflops / bf16_peak, 4),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)" if peaks_src == "measured"
                     else "fallback 1.59 PFLOP/s", "traffic": traffic,
                     "per_launch": "4*B*H*Npad*k*64*D executed flops (64x64 cube tiles of the k selected cubes)"},
        "wan720p_cfg_k64": cfg,
        "memory_kernels": {"workload": WORKLOAD, "peak_gbps": hbm_peak,
                           "peak_source": f"{peaks_src} HBM copy (MEASURED_PEAKS.json)", "kernels": mem},
        "pre_attention": {"api": "vsa_qk_norm_rope (Q/K RMSNorm over H*D + 3D RoPE), timed on its own, not in value",
                          "ms": round(pre_ms, 4), "bytes": pre_bytes, "bound": "hbm",
                          "achieved_gbps": round(pre_bytes / (pre_ms * 1e-3) / 1e9, 1), "peak_gbps": hbm_peak,
                          "frac": round(pre_bytes / (pre_ms * 1e-3) / 1e9 / hbm_peak, 4),
                          "per_launch": "Q and K read once and written once: 4*B*N*H*D*2 bytes"},
        "e2e": {"value": round(e2e_ms, 3), "unit": "ms", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "vsa_forward_host (pinned host q/k/v/gates in, host out; copies pipelined by head groups)"},
        # per step, VSA call: pool, coarse scores, coarse softmax x V, top-k, order sort, schedule, fine
        # (one-tile kernel) and the re-run guard (fine_kernel, which returns at once unless the one-tile
        # kernel overflowed) = 8; dense call: the one-tile kernel and its re-run guard = 2
        "gpu_launches": 10 * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "context": {"pages_dense_call_ms_b200": 17.0, "pages_vsa_kernel_ms_b200_k78": 4.719,
                    "pages_clip_s_b200": [133.0, 2.75]},
    }
    print(json.dumps(line), flush=True)


def run_stages(args):
    """Stage-by-stage times of one call on a named workload (rank 0 only, no process group)."""
    import torch

    import block_sparse_attention_cube_b200 as vsa
    w = synth.WORKLOADS[args.workload]
    x = synth.make_inputs(w)
    d = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in x.items()}
    ms = stage_times(vsa, torch, d, w, args.iters, 2, dense_too=args.dense_too, staged=args.staged)
    vsa.device_status()
    print(json.dumps({"workload": w.name, "iters": args.iters, "staged": args.staged, "ms": ms}), flush=True)


def run_calls(args):
    """`--iters` whole forward calls on a named workload (gated when it selects), each timed with events:
    a fixed case whose kernels a profiler can list one by one."""
    import torch

    import block_sparse_attention_cube_b200 as vsa
    w = synth.WORKLOADS[args.workload]
    x = synth.make_inputs(w)
    d = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in x.items()}
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    _, C = vsa.shape_info(s)
    gated = w.topk < C
    ws = vsa.alloc_workspace(s, w.topk)
    out = torch.empty_like(d["q"])
    stream = torch.cuda.current_stream()
    ms = []
    for _ in range(args.iters):
        e0, e1 = _events(torch, 2)
        e0.record(stream)
        vsa.forward(d["q"], d["k"], d["v"], s, w.topk, None, d["g_coarse"] if gated else None,
                    d["g_fine"] if gated else None, workspace=ws, out=out)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(round(e0.elapsed_time(e1), 4))
    vsa.device_status()
    print(json.dumps({"workload": w.name, "calls": args.iters, "ms": ms}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--stages", action="store_true", help="stage-by-stage times of one call (profiling case)")
    ap.add_argument("--calls", action="store_true", help="--iters whole forward calls on --workload (profiling case)")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synth.WORKLOADS), help="with --stages")
    ap.add_argument("--iters", type=int, default=3, help="with --stages")
    ap.add_argument("--dense-too", action="store_true", help="with --stages: add a dense fine-stage launch")
    ap.add_argument("--staged", action="store_true", help="with --stages: the unfused per-step entry points")
    args = ap.parse_args(argv)
    if args.stages:
        run_stages(args)
        return 0
    if args.calls:
        run_calls(args)
        return 0
    if args.warmup < 3 and args.impl == "cuda":
        ap.error("at least 3 warm-up steps")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_cuda(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
