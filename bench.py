"""Benchmark of the B200 VSA / dense attention path at the Wan 480p workload.

One step = one VSA call (grid 21x30x52 -> 39,936 padded tokens, 624 cubes,
40 heads, d=128, top-k 32 cubes, gated coarse + fine output) followed by one
dense attention call on the same Q/K/V (every cube selected, no gates), both
through the library's C ABI on one stream with inputs resident in HBM.

Prints one JSON line.  `value` is milliseconds per VSA call (whole job: with
N GPUs, N independent calls complete per step, so value = step time / N for
the VSA part); the dense call is reported beside it.  Timing: CUDA events on
the launching stream after warm-up, synchronize + barrier around the timed
region, max over ranks.  Inputs (1.0 GB of Q/K/V per call) exceed the 126 MB
L2, so L2 is not flushed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (extrapolated to one whole call) on rank 0 only.
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


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


# ---------------------------------------------------------------- the oracle arm
def oracle_sample(w, x, heads, cubes_per_head, seed=0):
    """Time the fp64 oracle on a bounded sample of workload `w` and extrapolate to one call.

    For each sampled head: tiling, pooling, coarse attention and top-k of the
    whole head, then the fine step for `cubes_per_head` query cubes and the
    merge / untiling of the head.  Returns (ms per call, seconds spent, sample text).
    """
    from oracle import vsa_oracle as O
    C = O.num_cubes(w.grid)
    scale = 1.0 / math.sqrt(w.head_dim)
    rng = np.random.default_rng(seed)
    cubes = sorted(rng.choice(C, size=min(cubes_per_head, C), replace=False).tolist())
    t_head = t_fine = 0.0
    for h in heads:
        f = {n: O.bf16_to_f64(x[n][:1, :, h:h + 1]) for n in x}
        t0 = time.perf_counter()
        qt, kt, vt = (O.tile(f[n], w.grid) for n in ("q", "k", "v"))
        if w.topk < C:
            bars = [O.pool(t, w.grid) for t in (qt, kt, vt)]
            scores, oc = O.coarse(*bars, scale)
            idx = O.topk(scores, w.topk)
        else:
            idx, oc = None, None
        t1 = time.perf_counter()
        o, _ = O.fine(qt, kt, vt, idx, scale, w.grid, items=[(0, 0, i) for i in cubes])
        t2 = time.perf_counter()
        o = np.nan_to_num(o)
        if oc is not None:
            o = O.combine(oc, o, f["g_coarse"], f["g_fine"], w.grid)
        O.untile(o, w.grid)
        t3 = time.perf_counter()
        t_head += (t1 - t0) + (t3 - t2)
        t_fine += t2 - t1
    nh = len(heads)
    per_call_s = w.batch * w.heads * (t_head / nh + (t_fine / nh) * C / len(cubes))
    sample = (f"{w.name}: heads {list(heads)} of {w.heads} (tile/pool/coarse/top-k/merge of each), fine step for "
              f"{len(cubes)} of {C} query cubes per head; extrapolated to {w.batch}x{w.heads} heads x {C} cubes")
    return per_call_s * 1e3, t_head + t_fine, sample


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
    # each step: one head, 32 query cubes (about a second of fp64 work)
    for _ in range(args.warmup):
        oracle_sample(w, x, heads=(0,), cubes_per_head=32, seed=0)
    vals, spent, sample = [], 0.0, ""
    for s in range(args.steps):
        ms, sec, sample = oracle_sample(w, x, heads=(s % w.heads,), cubes_per_head=32, seed=s)
        vals.append(ms)
        spent += sec
    value = statistics.mean(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "ms", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Philox, Wan 480p field inputs)",
        "config": {"workload": WORKLOAD, "batch": w.batch, "grid": "x".join(map(str, w.grid)), "heads": w.heads,
                   "head_dim": w.head_dim, "topk": w.topk},
        "cpu_baseline": {"value": round(value, 3), "unit": "ms", "cores": cores, "kind": "oracle",
                         "sample": sample + f" (one sampled head per step; {spent:.1f} s of CPU work in total)"},
        "e2e": {"value": round(value, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- the CUDA arm
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

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        vsa.forward(d["q"], d["k"], d["v"], s, w.topk, scale, d["g_coarse"], d["g_fine"], workspace=ws, out=out)
        if ev is not None:
            ev[1].record(stream)
        vsa.forward(d["q"], d["k"], d["v"], s, C, scale, workspace=ws_dense, out=out_d)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    vsa.device_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    vsa.device_status()
    step_ms = t_start.elapsed_time(t_end) / args.steps
    vsa_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    dense_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    step_ms_max = reduce_max(step_ms, world)
    vsa_ms_max = reduce_max(vsa_ms, world)
    dense_ms_max = reduce_max(dense_ms, world)

    # ---- per-stage breakdown: the launches of vsa_forward, one by one through the entry points
    names = ["pool", "coarse", "topk_order", "schedule", "fine"]
    acc = {n: [] for n in names}
    acc["fine_dense"] = []
    for it in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        e[0].record(stream)
        bars = vsa.pool_qkv(d["q"], d["k"], d["v"], s)
        e[1].record(stream)
        scores, oc = vsa.coarse(*bars, s, scale)
        e[2].record(stream)
        idx, order = vsa.topk_order(scores, s, w.topk)
        e[3].record(stream)
        steps = vsa.schedule(idx, s, order)
        e[4].record(stream)
        vsa.fine_fused(d["q"], d["k"], d["v"], s, idx, scale, order, oc, d["g_coarse"], d["g_fine"], out=out,
                       steps=steps)
        e[5].record(stream)
        vsa.fine_fused(d["q"], d["k"], d["v"], s, None, scale, out=out_d)
        e[6].record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            for j, n in enumerate(names):
                acc[n].append(e[j].elapsed_time(e[j + 1]))
            acc["fine_dense"].append(e[5].elapsed_time(e[6]))
        del bars, scores, oc, idx, order, steps
    stage_ms = {n: round(statistics.mean(v), 4) for n, v in acc.items()}

    # ---- the pre-attention pass (Q/K RMSNorm + 3D RoPE) on the same Q/K, timed on its own
    wts = synth.make_projection_inputs(synth.custom_workload("weights", 1, w.heads, w.head_dim, (1, 1, 1), 1))
    w_q, w_k = (torch.from_numpy(wts[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("w_q", "w_k"))
    q_n, k_n = torch.empty_like(d["q"]), torch.empty_like(d["k"])
    pre = []
    for it in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        vsa.qk_norm_rope(d["q"], d["k"], s, w_q, w_k, out=(q_n, k_n))
        e[1].record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            pre.append(e[0].elapsed_time(e[1]))
    pre_ms = reduce_max(statistics.mean(pre), world)
    del q_n, k_n

    # ---- end to end through vsa_forward_host (pinned host buffers, copies inside the timed region)
    h = {k: v.cpu().pin_memory() for k, v in d.items()}
    h_out = torch.empty_like(h["q"]).pin_memory()
    ws_host = vsa.alloc_workspace(s, w.topk, host_io=True, device=dev)
    for _ in range(max(1, args.warmup // 2)):
        vsa.forward_host(h["q"], h["k"], h["v"], s, w.topk, ws_host, h_out, scale, h["g_coarse"], h["g_fine"])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, args.steps // 2)
    e0.record(stream)
    for _ in range(e2e_steps):
        vsa.forward_host(h["q"], h["k"], h["v"], s, w.topk, ws_host, h_out, scale, h["g_coarse"], h["g_fine"])
    e1.record(stream)
    torch.cuda.synchronize()
    vsa.device_status()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, world)
    h2d = sum(h[k].numel() * 2 for k in ("q", "k", "v", "g_coarse", "g_fine"))
    d2h = h_out.numel() * 2

    if rank != 0:
        return
    peaks, peaks_src = load_peaks()
    bf16_peak = float(peaks["bf16_tflops"])
    hbm_peak = float(peaks["hbm_gbs"])
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
        ms_cpu, spent, sample = oracle_sample(w, x, heads=tuple(range(0, w.heads, 5)), cubes_per_head=320)
        cpu = {"value": round(ms_cpu, 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
               "sample": sample + f" ({spent:.1f} s of CPU work)"}
    line = {
        "metric": METRIC, "value": round(whole_job_ms_per_call(vsa_ms_max, 1, world), 4), "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox; Q/K = 0.5 N(0,1) + sin(0.3t+0.2x+0.1y+phi), V ~ N(0,1), gates U(0,1))",
        "config": {"workload": WORKLOAD, "batch": w.batch, "grid": "x".join(map(str, w.grid)),
                   "padded_tokens": npad, "cubes": C, "heads": w.heads, "head_dim": w.head_dim, "topk": w.topk,
                   "dense_call": {"workload": DENSE_WORKLOAD, "topk": C},
                   "l2": "no flush: 1.0 GB of Q/K/V per call exceeds the 126 MB L2",
                   "parallelism": f"{world} independent replicas (weak scaling)"},
        "dense_ms_per_call": round(whole_job_ms_per_call(dense_ms_max, 1, world), 4),
        "stage_ms": stage_ms,
        "fine": {"executed_tflop": round(fine_flops / 1e12, 4), "tflops": round(fine_tflops, 1),
                 "frac_bf16_peak": round(fine_tflops / bf16_peak, 4),
                 "dense_equivalent_tflops": round(dense_equivalent_flops(w.batch, w.heads, w.tokens, w.head_dim)
                                                  / (stage_ms["fine"] * 1e-3) / 1e12, 1)},
        "dense_fine": {"executed_tflop": round(dense_flops / 1e12, 3), "tflops": round(dense_tflops, 1),
                       "frac_bf16_peak": round(dense_tflops / bf16_peak, 4),
                       "per_launch": "4*B*H*(64*ceil(N/64))^2*D: blocks of 64 real tokens, no padding"},
        "roofline": {"kernel": "fine_tile_kernel<128, cubes> (VSA, top-k 32)", "bound": "tensor",
                     "achieved": round(fine_tflops, 2),
                     "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(fine_tflops / bf16_peak, 4),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)" if peaks_src == "measured"
                     else "fallback 1.59 PFLOP/s", "traffic": traffic,
                     "per_launch": "4*B*H*Npad*k*64*D executed flops (64x64 cube tiles of the k selected cubes)"},
        "pre_attention": {"api": "vsa_qk_norm_rope (Q/K RMSNorm over H*D + 3D RoPE), timed on its own, not in value",
                          "ms": round(pre_ms, 4), "bytes": pre_bytes, "bound": "hbm",
                          "achieved_gbps": round(pre_bytes / (pre_ms * 1e-3) / 1e9, 1), "peak_gbps": hbm_peak,
                          "frac": round(pre_bytes / (pre_ms * 1e-3) / 1e9 / hbm_peak, 4),
                          "per_launch": "Q and K read once and written once: 4*B*N*H*D*2 bytes"},
        "e2e": {"value": round(e2e_ms, 3), "unit": "ms", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "vsa_forward_host (pinned host q/k/v/gates in, host out; copies pipelined by head groups)"},
        # per step, VSA call: pool, coarse scores, coarse softmax x V, top-k, order sort, schedule, fine
        # (one-tile kernel) and the re-run guard (fine_kernel, which returns at once unless the one-tile
        # kernel overflowed) = 8; dense call: fine = 1
        "gpu_launches": 9 * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "context": {"pages_dense_call_ms_b200": 17.0, "pages_vsa_kernel_ms_b200_k78": 4.719,
                    "pages_clip_s_b200": [133.0, 2.75]},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    args = ap.parse_args(argv)
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
