"""bench.py's multi-rank plumbing on CPU: world size 2 over gloo (127.0.0.1).

Each rank contributes its own timing; the slowest rank's time and the
whole-job aggregate must come out identical on every rank, and the reference
arm must print only on rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, l = bench.dist_env()
    assert (r, w, l) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    t_max = bench.max_over_ranks(1.0 + rank, w, "cpu")
    value = bench.aggregate(3e12, t_max, w)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, t_max, value))


def test_max_over_ranks_and_aggregate_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r for r, _, _ in res] == [0, 1]
    for _, t_max, value in res:
        assert t_max == 2.0                      # the slowest rank
        assert value == pytest.approx(3.0)      # 2 ranks x 3e12 flop / 2 s = 3 TFLOP/s


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _dying_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import time
    import bench
    bench.dist_init(world, "gloo")
    bench.barrier(world)
    if rank == 1:
        os._exit(3)  # a rank that dies between steps, without leaving the group
    time.sleep(1.0)
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0, world, "cpu")
        q.put((rank, "completed", time.monotonic() - t0))
    except Exception as e:  # the collective must end with an error, not wait
        q.put((rank, type(e).__name__, time.monotonic() - t0))
    # Flush the queue's feeder thread before leaving without the process
    # group's normal shutdown (which would wait on the dead peer).
    q.close()
    q.join_thread()
    os._exit(0)


def test_a_dead_rank_ends_the_next_collective_with_an_error():
    """Failure detection on the host: rank 1 dies between steps; rank 0's next
    timing all-reduce fails with an error within the process group's timeout
    instead of waiting for ever."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=200)
    assert procs[1].exitcode == 3
    assert procs[0].exitcode == 0, "rank 0 did not come back from its collective"
    rank, outcome, waited = q.get(timeout=10)
    assert rank == 0 and outcome != "completed", outcome
    assert waited < 130
