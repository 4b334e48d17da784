"""Benchmark of the rotation + INT4 W4A4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload q_proj]

One step = one pass of the whole path over one batch: pq_transform_quant(X) (rotate +
quantise the activations), pq_pack_weights(W) (rotate + quantise the weights), pq_w4a4_gemm
(codes -> Y float32).  Default workload: the block-Hadamard q_proj shape, X bf16 [2048, 4096],
W bf16 [4096, 4096], g = 128 (synthetic, seeded).  L2 is flushed (256 MiB write, then a 256 MiB read) between timed
steps; each step is timed with CUDA events on the launching stream, and the sum over K steps is
reduced with MAX over ranks.  N > 1 runs independent replicas (no data-path collective):
``scaling`` is weak and ``value`` is the total over ranks.

The reference arm (``--impl reference``) times the CPU oracle on this machine's host cores on a
bounded sample of the same workload, extrapolated to a full step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "rotate+quant GB/s (% HBM peak); W4A4 GEMM TOPS (% INT8 tensor peak)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Nominal dense ratio of the contraction's tensor dtype to bf16: the GEMM's MMAs are E4M3
# (kind::f8f6f4), 4.5 PFLOP/s dense like int8's 4.5 POPS, against 2.25 PFLOP/s for bf16.
INT8_OVER_BF16 = 4.5 / 2.25
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 1000 * 1000                     # B200 L2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(wl):
    """Algorithmic bytes / ops per kernel launch for the workload."""
    T, D, N, g = wl.T, wl.D, wl.N, wl.g
    per_elem = 2 + 0.5 + 4.0 / g                     # bf16 in, nibble out, one f32 scale / group
    smooth = 4.0 / g if wl.kind == "smooth_hadamard" else 0.0
    return {
        "transform_quant_bytes": T * D * (per_elem + smooth),
        "pack_weights_bytes": N * D * per_elem,
        "gemm_ops": 2.0 * T * N * D,
        "gemm_bytes": T * D / 2 + N * D / 2 + (T + N) * (D // g) * 4 + T * N * 4,
    }


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.lines: list[tuple[float, str]] = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, x_rows=128, w_rows=1024):
    """Time the oracle on a bounded sample and extrapolate to one full step (seconds)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    plan = oracle.Plan(wl.kind, wl.D, wl.g, wl.K, None, wl.angles, wl.beta)
    if wl.kind == "givens":
        plan.pairs = oracle.select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, wl.g // 2)
    xs = wl.X[:max(x_rows, 128) if wl.kind == "smooth_hadamard" else x_rows]
    ws = wl.W[:w_rows]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        a = oracle.transform_quant(xs, plan)
        t1 = time.perf_counter()
        w = oracle.pack_weights(ws, plan)
        t2 = time.perf_counter()
        oracle.gemm(a.codes, a.scales, w.codes, w.scales, wl.g)
        t3 = time.perf_counter()
    xr = xs.shape[0]
    full = (t1 - t0) * wl.T / xr + (t2 - t1) * wl.N / w_rows + (t3 - t2) * (wl.T / xr) * (wl.N / w_rows)
    sample = (f"oracle (numpy float64, 1 thread) on X rows 0..{xr - 1} and W rows 0..{w_rows - 1}: "
              f"transform {t1 - t0:.3f}s, weight pack {t2 - t1:.3f}s, GEMM {t3 - t2:.3f}s, "
              f"extrapolated linearly to T={wl.T}, N={wl.N}")
    return full, t3 - t0, sample


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    steps = []
    for i in range(args.warmup + args.steps):
        full, spent, sample = oracle_sample(wl)
        if i >= args.warmup:
            steps.append(full)
    total = sum(steps)
    value = wl.T * len(steps) / total
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (oracle)", "data": "synthetic (seeded)", "config": config_of(wl, "n/a"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(wl, l2):
    return {"workload": f"{wl.name}: {wl.description}; W bf16 [{wl.N},{wl.D}] N(0,0.02); g={wl.g}",
            "T": wl.T, "D": wl.D, "N": wl.N, "g": wl.g, "K_layers": wl.K, "kind": wl.kind,
            "out": "float32", "l2": l2, "parallelism": "replicas (one independent workload per GPU)"}


def max_over_ranks(x, world, device):
    """Max of a per-rank float over all ranks (the process group's backend: NCCL on the GPU
    arm, gloo in the CPU tests).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, tokens_per_rank_step, steps, total_ms):
    """Whole-job tokens/s: every rank processes its own workload (weak scaling); the slowest
    rank's device time bounds the job."""
    return world * tokens_per_rank_step * steps / (total_ms * 1e-3)


# Kernels one step launches: transform_quant and pack_weights (one each), then the GEMM's own
# launches as the library reports them for these sizes on the current device (operand
# expansion and contraction, plus the split-K reduction when it splits the group range).
LAUNCHES_PER_STEP = 4


def launches_per_step(T, N, D):
    from rotation_int4_w4a4_b200 import pq
    return 2 + pq.pq_w4a4_gemm_launch_count(T, N, D)


# ------------------------------------------------------------------------ GPU arm
def run_ours(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from rotation_int4_w4a4_b200 import pq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    kind = wl.kind
    if kind == "givens":
        pairs = pq.pq_select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, wl.g // 2)
        plan = pq.Plan("givens", wl.D, K=wl.K, pairs=pairs, angles=wl.angles, beta=wl.beta)
    else:
        plan = pq.Plan(kind, wl.D)
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // wl.g
    X0, W0 = dev_bf16(wl.X), dev_bf16(wl.W)
    smooth_w = torch.ones(D, dtype=torch.float32, device=dev) if kind == "smooth_hadamard" else None

    def buffer_set(first):
        return {"X": X0 if first else X0.clone(), "W": W0 if first else W0.clone(),
                "ca": torch.empty((T, D // 2), dtype=torch.uint8, device=dev),
                "sa": torch.empty((T, G), dtype=torch.float32, device=dev),
                "cw": torch.empty((N, D // 2), dtype=torch.uint8, device=dev),
                "sw": torch.empty((N, G), dtype=torch.float32, device=dev),
                "Y": torch.empty((T, N), dtype=torch.float32, device=dev),
                "sm": torch.empty(((T + 127) // 128, D), dtype=torch.float32, device=dev)
                if kind == "smooth_hadamard" else None}

    # Cold L2 between steps.  "flush" (default): one set of buffers, and a 256 MiB write + read
    # between steps.  "rotate": enough complete sets of inputs and outputs that a step's buffers
    # were last touched over 2 x L2 bytes ago and no other kernel runs between steps (the previous
    # step's dirty outputs are then written back during the next step).
    footprint = sum(t.numel() * t.element_size() for t in buffer_set(True).values() if t is not None)
    nsets = 1 if args.l2 == "flush" else max(2, -(-2 * L2_BYTES // footprint))
    sets = [buffer_set(i == 0) for i in range(nsets)]
    flush = L2Flush(dev) if args.l2 == "flush" else (lambda: None)
    l2_desc = (f"flushed between steps (256 MiB write, then 256 MiB read)" if args.l2 == "flush" else
               f"cold: {nsets} rotating sets of inputs and outputs ({nsets * footprint / 1e6:.0f} MB "
               f"working set, > 2 x the 126 MB L2); no other kernel between steps")

    def run_step(bs):
        pq.pq_transform_quant(plan, bs["X"], bs["ca"], bs["sa"], bs["sm"], stream=stream)
        pq.pq_pack_weights(plan, bs["W"], bs["cw"], bs["sw"], smooth_w, stream=stream)
        pq.pq_w4a4_gemm(bs["ca"], bs["sa"], bs["cw"], bs["sw"], bs["Y"], stream=stream)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def timed_step(k):
        bs = sets[(k + offset) % nsets]
        e = ev[k]
        e[0].record(stream)
        pq.pq_transform_quant(plan, bs["X"], bs["ca"], bs["sa"], bs["sm"], stream=stream)
        e[1].record(stream)
        pq.pq_pack_weights(plan, bs["W"], bs["cw"], bs["sw"], smooth_w, stream=stream)
        e[2].record(stream)
        pq.pq_w4a4_gemm(bs["ca"], bs["sa"], bs["cw"], bs["sw"], bs["Y"], stream=stream)
        e[3].record(stream)

    for i in range(args.warmup):
        flush()
        run_step(sets[i % nsets])
    torch.cuda.synchronize()
    pq.pq_check_status(plan)

    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(vis[local_rank] if local_rank < len(vis) else str(local_rank))
    clocks.start()
    t_roll = time.time()
    i = 0
    while time.time() - t_roll < 0.6:            # keep the GPU busy while sampling starts
        flush()
        run_step(sets[i % nsets])
        i += 1
        torch.cuda.synchronize()
    offset = i                                   # the first timed step uses the least recent set

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    for k in range(args.steps):
        flush()
        timed_step(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    w1 = time.time()
    t_post = time.time()
    while time.time() - t_post < 0.4:
        flush()
        run_step(sets[i % nsets])
        i += 1
        torch.cuda.synchronize()
    clocks.stop()
    pq.pq_check_status(plan)

    per = [[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in ev]     # ms
    step_ms = [sum(p) for p in per]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    tq_ms = statistics.mean(p[0] for p in per)
    pw_ms = statistics.mean(p[1] for p in per)
    gm_ms = statistics.mean(p[2] for p in per)

    # ---------------------------------------------------------------- end to end
    e2e_ms, h2d, d2h = e2e_run(args, wl, pq, plan, dev, stream, flush, sets[0]["sm"], smooth_w)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    alg = algorithmic(wl)
    hbm = peaks["hbm_gbs"]
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    comps = {
        "transform_quant": {"us": 1e3 * tq_ms, "GB_s": alg["transform_quant_bytes"] / (tq_ms * 1e-3) / 1e9},
        "pack_weights": {"us": 1e3 * pw_ms, "GB_s": alg["pack_weights_bytes"] / (pw_ms * 1e-3) / 1e9},
        "w4a4_gemm": {"us": 1e3 * gm_ms, "TOPS": alg["gemm_ops"] / (gm_ms * 1e-3) / 1e12},
    }
    comps["transform_quant"]["frac_hbm"] = comps["transform_quant"]["GB_s"] / hbm
    comps["pack_weights"]["frac_hbm"] = comps["pack_weights"]["GB_s"] / hbm
    comps["w4a4_gemm"]["frac_int8"] = comps["w4a4_gemm"]["TOPS"] / int8_peak
    dominant = max(("transform_quant", tq_ms), ("pack_weights", pw_ms), ("w4a4_gemm", gm_ms), key=lambda kv: kv[1])[0]
    traffic = load_traffic(dominant, wl)
    if dominant == "w4a4_gemm":
        roof = {"bound": "tensor", "achieved": comps[dominant]["TOPS"], "peak": int8_peak, "unit": "TOPS",
                "frac": comps[dominant]["TOPS"] / int8_peak, "traffic": traffic, "kernel": dominant,
                "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {INT8_OVER_BF16} "
                               "(nominal dense fp8 = int8 : bf16 ratio; the MMAs are E4M3)",
                "algorithmic": f"2*T*N*D = {alg['gemm_ops']:.4g} ops per launch"}
    else:
        roof = {"bound": "hbm", "achieved": comps[dominant]["GB_s"], "peak": hbm, "unit": "GB/s",
                "frac": comps[dominant]["GB_s"] / hbm, "traffic": traffic, "kernel": dominant,
                "peak_source": f"{peak_src} copy bandwidth"}
    value = job_value(world, wl.T, args.steps, total_ms)
    cpu = None
    if world == 1:
        full, spent, sample = oracle_sample(wl)
        cpu = {"value": wl.T / full, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample}
    ck = clocks.summary(t_roll, time.time())
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in; f32 transform; e4m3 MMA -> f32; f32 out",
            "data": "synthetic (seeded SplitMix64 generator)",
            "config": config_of(wl, l2_desc),
            "components": comps, "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": job_value(world, wl.T, 1, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step(wl.T, wl.N, wl.D) * args.steps, "clocks": ck, "wall_s_timed_region": w1 - w0}
    print(json.dumps(line), flush=True)


def e2e_run(args, wl, pq, plan, dev, stream, flush, sm, smooth_w):
    """Same step through the public API from pinned host buffers: H2D of X and W, the three
    calls, D2H of Y, all inside the CUDA-event-timed region."""
    import numpy as np
    import torch
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // wl.g
    hX = torch.from_numpy(np.ascontiguousarray(wl.X).view(np.int16)).pin_memory()
    hW = torch.from_numpy(np.ascontiguousarray(wl.W).view(np.int16)).pin_memory()
    hY = torch.empty((T, N), dtype=torch.float32).pin_memory()
    dX = torch.empty((T, D), dtype=torch.int16, device=dev)
    dW = torch.empty((N, D), dtype=torch.int16, device=dev)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)
    total = 0.0
    n = max(3, min(args.steps, 10))
    for i in range(args.warmup + n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        dX.copy_(hX, non_blocking=True)
        dW.copy_(hW, non_blocking=True)
        pq.pq_transform_quant(plan, dX, ca, sa, sm, T=T, ldx=D, stream=stream)
        pq.pq_pack_weights(plan, dW, cw, sw, smooth_w, N=N, stream=stream)
        pq.pq_w4a4_gemm(ca, sa, cw, sw, Y, stream=stream)
        hY.copy_(Y, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            total += e0.elapsed_time(e1)
    pq.pq_check_status(plan)
    return total / n, hX.numel() * 2 + hW.numel() * 2, hY.numel() * 4


class L2Flush:
    """Evicts this GPU's L2 between timed steps: writes a 256 MiB buffer (twice the 126 MB L2),
    then reads another 256 MiB buffer so that the write's dirty lines are written back before
    the next timed kernel instead of during it."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.out)


def load_traffic(kernel, wl):
    """DRAM bytes per launch from the committed ncu summary for this kernel and workload, if any."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return d.get(f"{kernel}:{wl.name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q_proj")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--N", type=int, default=None, help="sweep workload: 4096 or 14336")
    ap.add_argument("--kind", default=None, help="sweep workload: hadamard or givens")
    ap.add_argument("--l2", choices=["flush", "rotate"], default="flush",
                    help="cold L2 between steps: a 256 MiB write + read (default), or rotating sets "
                         "of inputs and outputs larger than twice the L2")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from rotation_int4_w4a4_b200 import inputs
    wl = inputs.workload(args.workload, T=args.T, N=args.N, kind=args.kind)

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
