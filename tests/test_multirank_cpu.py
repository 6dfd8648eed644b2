"""The benchmark's N > 1 host logic on CPU: two gloo ranks (world size 2).

Under torchrun every rank runs its own replica batch (the decode path has no
exchange step), the job time is the slowest rank's, and the job rate counts
every rank's queries.  The reference arm runs on rank 0 alone.  These checks
run the same helpers bench.py uses, with gloo in place of NCCL.
"""
import hashlib
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

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
    w, r, _ = bench.dist_init("gloo")
    own_time = 1.0 + 0.5 * r                      # rank 1 is the slow one
    t_max = bench.max_over_ranks(own_time, w)
    bench.barrier(w)
    inp = bench.replica_inputs(1, r)
    digest = hashlib.sha256(inp.q_idx.tobytes() + inp.kidx.tobytes()).hexdigest()
    rate = bench.job_rate(inp.nq, 10, w, t_max)
    args = type("A", (), {"workload": "tiny_decode_4k", "warmup": 1, "steps": 1})()
    ref = bench.run_reference(args, w, r)
    out.put((r, w, t_max, digest, inp.nq, rate, ref))
    dist.destroy_process_group()


@pytest.fixture(scope="module")
def results():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r, *rest = q.get(timeout=120)
        res[r] = rest
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_ranks_agree_on_the_slowest_time(results):
    assert results[0][0] == results[1][0] == 2
    assert results[0][1] == results[1][1] == pytest.approx(1.5)


def test_replicas_draw_their_own_inputs(results):
    assert results[0][2] != results[1][2]
    assert results[0][3] == results[1][3]          # same shape on every rank


def test_job_rate_counts_every_rank(results):
    nq = results[0][3]
    assert results[0][4] == pytest.approx(nq * 10 * 2 / 1.5)


def test_reference_arm_runs_on_rank_zero_only(results):
    assert results[1][5] is None                   # rank 1 does no work and prints nothing
    line = results[0][5]                           # rank 0 times the oracle and returns its line
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "queries/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "tiny_decode_4k"
