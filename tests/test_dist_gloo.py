"""Host logic of the multi-process benchmark on CPU: two ranks over gloo.

The decode path does not shard (every rank is an independent replica), so the
only cross-rank operations are the host-side timing reductions and barriers of
bench.py, and the rank-0-only output of the launch contract.  These run here
as world_size-2 process groups on 127.0.0.1.
"""

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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, w, _ = bench.dist_init()
    assert (r, w) == (rank, world) and dist.get_backend() == "gloo"
    bench.barrier()
    mx = bench.max_over_ranks(10.0 + rank)          # each rank's time; the job's time is the max
    sm = bench.sum_over_ranks(100.0 * (rank + 1))   # units processed by all ranks
    ref = bench.run_reference(type("A", (), {"gpus": world, "steps": 1, "warmup": 0})(),
                              bench.workload_spec("tiny_g2"), rank)
    out.put((rank, mx, sm, ref is None))
    bench.barrier()
    dist.destroy_process_group()


def test_timing_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]          # max over ranks on every rank
    assert [r[2] for r in res] == [300.0, 300.0]        # sum over ranks on every rank
    assert [r[3] for r in res] == [False, True]         # the reference arm runs on rank 0 only


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny_g2", "--steps", "1", "--warmup", "1", "--gpus", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
