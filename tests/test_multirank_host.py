"""The multi-GPU bench path's host logic on CPU: two gloo ranks.

Decode attention shards by sequence with no data exchange, so N GPUs run N
independent replicas; the only collectives are the barrier and the max of the
per-rank step times.  Those, the per-rank seeds, the whole-job aggregation and
the reference arm's rank handling are checked here without a GPU."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, loc = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w)
    try:
        step_ms = [1.25, 3.5][r]  # rank 1 is the slow one
        slowest = bench.max_over_ranks(step_ms, w)
        dist.barrier()

        class Args:  # the reference arm's arguments, smallest bounded sample
            gpus, steps, warmup, workload = w, 1, 0, "gemma4_12b_stack_b8_l8192"
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.run_reference(Args, w, r) if r == 1 else 0
        out_q.put((r, slowest, bench.rank_seed_offset(r), rc, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [3.5, 3.5]          # both ranks see the max
    assert res[0][2] != res[1][2]                     # distinct sequence seeds
    assert res[1][3] == 0 and res[1][4] == ""         # reference arm: rank 1 prints nothing


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    per_rank = 3 * 2 ** 30
    one = bench.job_gbs(per_rank, 0.8, 1)
    assert bench.job_gbs(per_rank, 0.8, 2) == pytest.approx(2 * one)   # weak scaling
    assert bench.job_gbs(per_rank, 1.6, 2) == pytest.approx(one)       # slowest rank rules
    assert one == pytest.approx(per_rank / 0.8e-3 / 1e9)


def test_reference_arm_prints_one_json_line_on_rank0():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        gpus, steps, warmup, workload = 1, 1, 0, "gemma4_12b_stack_b8_l8192"
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(Args, 1, 0) == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
