"""Run one workload's hot-path step a few times through the library, for profilers.

    python profile_step.py [--workload q_proj] [--T tokens] [--N rows] [--repeat 3] [--rrs]

Each repetition launches, in order, the activation transform (pq_transform_quant), the weight
transform (pq_pack_weights) and the W4A4 GEMM (pq_w4a4_gemm) on the named synthetic workload,
then checks the device status.  With --rrs it runs rotated runtime smoothing on the workload's
shapes instead (pq_rrs_prepare, pq_rrs_transform_quant, pq_rrs_pack_weights, pq_rrs_gemm; a
block-Hadamard plan).  Nothing else runs on the GPU, so a profiler's kernel filter and
launch skip select launches by position (e.g. -s 4 skips the first repetition of a 4-launch
step).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main() -> None:
    import torch

    from rotation_int4_w4a4_b200 import inputs, pq

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="q_proj")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--N", type=int, default=None)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--rrs", action="store_true")
    args = ap.parse_args()
    wl = inputs.workload(args.workload, T=args.T, N=args.N)
    dev = torch.device("cuda")

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    X, W = bf16(wl.X), bf16(wl.W)
    if args.rrs:
        run_rrs(wl, X, W, args.repeat, dev)
        return
    if wl.kind == "givens":
        pairs = pq.pq_select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, wl.g // 2)
        plan = pq.Plan("givens", wl.D, K=wl.K, pairs=pairs, angles=wl.angles, beta=wl.beta)
    else:
        plan = pq.Plan(wl.kind, wl.D)
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // wl.g
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)
    smooth = wl.kind == "smooth_hadamard"
    sm = torch.empty(((T + 127) // 128, D), dtype=torch.float32, device=dev) if smooth else None
    smooth_w = torch.ones(D, dtype=torch.float32, device=dev) if smooth else None
    for _ in range(args.repeat):
        pq.pq_transform_quant(plan, X, ca, sa, sm)
        pq.pq_pack_weights(plan, W, cw, sw, smooth_w)
        pq.pq_w4a4_gemm(ca, sa, cw, sw, Y)
    pq.pq_check_status(plan)
    print(f"{wl.name}: {args.repeat} steps, Y[0, :4] = {Y[0, :4].tolist()}")


def run_rrs(wl, X, W, repeat, dev) -> None:
    import torch

    from rotation_int4_w4a4_b200 import pq
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // wl.g
    plan = pq.Plan("hadamard", D)
    f32, i32, u8 = torch.float32, torch.int32, torch.uint8
    cm, gs = torch.empty(D, dtype=f32, device=dev), torch.empty(G, dtype=f32, device=dev)
    perm, inv = torch.empty(D, dtype=i32, device=dev), torch.empty(D, dtype=i32, device=dev)
    ca, ts = torch.empty((T, D // 2), dtype=u8, device=dev), torch.empty(T, dtype=f32, device=dev)
    cw, sw = torch.empty((N, D // 2), dtype=u8, device=dev), torch.empty((N, G), dtype=f32, device=dev)
    Y = torch.empty((T, N), dtype=f32, device=dev)
    for _ in range(repeat):
        pq.pq_rrs_prepare(plan, X, cm, perm, inv, gs)
        pq.pq_rrs_transform_quant(plan, X, perm, gs, ca, ts)
        pq.pq_rrs_pack_weights(plan, W, perm, gs, cw, sw)
        pq.pq_rrs_gemm(ca, ts, cw, sw, Y)
    pq.pq_check_status(plan)
    print(f"{wl.name} (rrs): {repeat} steps, Y[0, :4] = {Y[0, :4].tolist()}")


if __name__ == "__main__":
    main()
