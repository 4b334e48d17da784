"""Host logic of bench.py's multi-rank path, on CPU with two gloo ranks.

The GPU arm runs one independent workload per rank (replicas, weak scaling).  Its only
collectives are the barriers around the timed region and the max-over-ranks reduction of the
device times; the reference arm runs on rank 0 alone.  These tests run those pieces with the
gloo backend on 127.0.0.1.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # each rank reports a different device time; every rank must see the slowest one
        mine = 10.0 + 7.5 * rank
        dist.barrier()
        got = bench.max_over_ranks(mine, world, "cpu")
        value = bench.job_value(world, 2048, 20, got)
        # reference arm: only rank 0 prints its JSON line
        args = type("A", (), {"warmup": 0, "steps": 1})()
        from rotation_int4_w4a4_b200 import inputs
        wl = inputs.workload("tiny")
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(args, wl, rank, world, workers=2)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "value": value, "stdout": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_reference_on_rank0(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["max"] for r in res] == [17.5, 17.5]
    # whole-job tokens/s: both ranks' tokens over the slowest rank's time
    assert res[0]["value"] == pytest.approx(2 * 2048 * 20 / 17.5e-3)
    assert res[1]["stdout"] == ""
    lines = [l for l in res[0]["stdout"].splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    for key in ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "higher_is_better",
                "cpu_baseline", "e2e", "config"):
        assert key in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_job_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_value(1, 2048, 10, 5.0)
    assert bench.job_value(4, 2048, 10, 5.0) == pytest.approx(4 * one)
    assert bench.LAUNCHES_PER_STEP == 4
    # No GPU here: the library counts with B200's 148 SMs (74 SM pairs).
    assert bench.launches_per_step(2048, 4096, 4096) == 4      # 128 pair tiles: no split
    assert bench.launches_per_step(256, 4096, 4096) == 5       # 16 pair tiles: split-K + reduce
    assert bench.launches_per_step(1, 4096, 4096) == 3         # at most 4 tokens: CUDA-core kernel
    assert bench.launches_per_step(4, 14336, 4096) == 3
    assert bench.launches_per_step(16, 4096, 4096) == 4        # few tokens: group ranges + reduce
    assert bench.launches_per_step(17, 14336, 4096) == 3       # few tokens, 112 tiles: one launch
    assert bench.launches_per_step(64, 4096, 4096) == 4        # few tokens: ranges + reduce
    assert bench.launches_per_step(17, 272, 4096) == 4         # ragged N: ranges + reduce


def test_e2e_chunks_keep_the_whole_calls_kernels():
    """The end-to-end step splits the tokens only where every chunk's GEMM takes the same kernels
    as the whole call (no split-K the whole call would not make), in whole 256-token tiles."""
    sys.path.insert(0, ROOT)
    import bench
    from rotation_int4_w4a4_b200 import pq
    for T, N, D in ((8192, 4096, 14336), (4096, 14336, 4096), (2048, 4096, 4096), (16384, 4096, 4096),
                    (1000, 4096, 4096), (1, 4096, 4096), (8200, 4096, 14336)):
        chunks = bench.e2e_chunks(T, N, D)
        assert chunks[0][0] == 0 and chunks[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(chunks, chunks[1:]))
        assert all(t0 % 256 == 0 for t0, _ in chunks)
        whole = pq.pq_w4a4_gemm_launch_count(T, N, D)
        assert all(pq.pq_w4a4_gemm_launch_count(t1 - t0, N, D) == whole for t0, t1 in chunks)
    assert len(bench.e2e_chunks(8192, 4096, 14336)) == 8          # the default workload
    assert bench.e2e_chunks(2048, 4096, 4096) == [(0, 2048)]      # 512-token chunks would split K
