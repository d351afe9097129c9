"""Host logic of the N-rank benchmark, as two gloo ranks on CPU.

The benchmark runs one process per GPU; every rank holds a replica of the
index and searches its own query batch, the job's time is the slowest rank's
device time, and only rank 0 prints.  These tests run that logic (process
group, max over ranks, whole-job throughput, per-rank batches) with world
size 2 on the CPU, and the reference arm under torchrun.
"""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, nproc=2, timeout=300):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", *args]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    return subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)


WORKER = textwrap.dedent("""
    import json, os, sys
    sys.path.insert(0, {root!r})
    import numpy as np, torch, torch.distributed as dist
    import bench
    from mips_ivf_centroid_b200 import datagen
    rank, world, local = bench.dist_env()
    dev = torch.device("cpu")
    assert bench.init_ranks(world, dev)
    # a rank's device time: rank 1 is the slow one
    mine = 100.0 + 50.0 * rank
    slowest = bench.max_over_ranks(mine, dev, world)
    value, ms = bench.job_throughput(world, 1000, slowest, 10)
    w = datagen.WORKLOADS["tiny"].scaled(nq=8)
    q = datagen.make_queries(bench.rank_workload(w, rank))
    first = torch.from_numpy(np.ascontiguousarray(q[0]))
    got = [torch.empty_like(first) for _ in range(world)]
    dist.all_gather(got, first)
    dist.barrier()
    out = dict(rank=rank, world=world, slowest=slowest, value=value, ms=ms,
               same_batch=bool(torch.equal(got[0], got[1])),
               q0=q[0].tolist()[:4])
    with open(os.path.join({tmp!r}, f"rank{{rank}}.json"), "w") as f:
        json.dump(out, f)
    dist.destroy_process_group()
""")


def test_two_ranks_time_is_the_slowest_and_value_counts_every_rank(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT, tmp=str(tmp_path)))
    r = _torchrun([str(script)])
    assert r.returncode == 0, r.stderr[-2000:]
    res = [json.loads((tmp_path / f"rank{i}.json").read_text()) for i in range(2)]
    for x in res:
        assert x["world"] == 2
        assert x["slowest"] == 150.0                       # max over ranks, on every rank
        assert x["ms"] == pytest.approx(15.0)              # 150 ms over 10 steps
        assert x["value"] == pytest.approx(2 * 1000 / 15e-3)
        assert not x["same_batch"]                         # each rank its own queries
    # a rank's batch is a function of its rank only
    from mips_ivf_centroid_b200 import datagen
    import bench
    w = datagen.WORKLOADS["tiny"].scaled(nq=8)
    for x in res:
        q = datagen.make_queries(bench.rank_workload(w, x["rank"]))
        assert q[0].tolist()[:4] == pytest.approx(x["q0"], abs=0)


def test_single_rank_needs_no_process_group():
    import torch
    import bench
    assert not bench.init_ranks(1, torch.device("cpu"))
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    v, ms = bench.job_throughput(1, 1000, 40.0, 100)
    assert ms == pytest.approx(0.4) and v == pytest.approx(1000 / 0.4e-3)


def test_reference_arm_prints_once_under_two_ranks():
    r = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny",
                   "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cpu_model"] and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
