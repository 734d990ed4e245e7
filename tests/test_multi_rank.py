"""The benchmark's multi-process logic on the CPU with gloo, world size 2: every rank
meets at the barriers, the elapsed time is the max over ranks, the whole-job value
counts every rank's units, and the reference arm runs on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    bench.barrier(w)
    ms = bench.max_over_ranks(1.0 + rank, w)          # rank 1 is the slowest
    value = bench.aggregate(1e9, ms, w)              # 1 GB per rank
    dist.destroy_process_group()
    q.put((rank, ms, value))


def test_max_over_ranks_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in res:
        assert ms == 2.0                                 # max over ranks, on every rank
        assert abs(value - 2 * 1e9 / 2e-3) < 1e-3        # units of both ranks / slowest time


def _ref_worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "3",
                "--workload", "decode64", "--cpu-budget", "0.5"]
    buf = io.StringIO()
    if rank == 0:
        # keep the reference arm short: time one tiny decode workload instead of decode64
        from gated_deltanet_recurrent_la_b200 import workloads as W
        W.WORKLOADS["decode64"] = lambda seed=0: W.step_inputs(B=2, n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16,
                                                               n_slots=4, seed=seed)
    with redirect_stdout(buf):
        rc = bench.main()
    q.put((rank, rc, buf.getvalue()))


def test_reference_arm_prints_on_rank0_only():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_ref_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert res[0][1] == 0 and res[1][1] == 0
    assert res[1][2] == ""                                # other ranks exit without work
    line = json.loads(res[0][2].strip())
    assert line["impl"] == "reference" and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
