"""CPU tests of bench.py's multi-rank host logic (replicas only): two gloo
ranks on 127.0.0.1.

- the timed figures are the slowest rank's (max over ranks), taken in the
  same order on every rank;
- the job's time per token divides by every rank's tokens;
- the reference arm runs on rank 0 only; the other ranks exit 0 at once.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # every rank measured a different device time; all see the slowest
        a = bench.max_over_ranks(10.0 + 3.5 * rank, world, "cpu")
        b = bench.max_over_ranks(7.0 - rank, world, "cpu")
        out[rank] = (a, b, bench.job_ms_per_token(a, 4, world))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        a, b, v = out[r]
        assert a == 13.5 and b == 7.0
        assert v == pytest.approx(13.5 / (4 * 2))


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_ms_per_token(8.0, 4, 1) == 2.0


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank0_only(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        rec = json.loads(lines[0])
        assert rec["impl"] == "reference" and rec["n_gpus"] == 2
        assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
        assert rec["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []
