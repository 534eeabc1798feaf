"""The multi-rank host paths of bench.py on CPU with gloo, world size 2.

bench.py runs one replica per GPU (sequences are independent; no collective in
the timed region): the only cross-rank steps are barriers around the timed
region and the max over ranks of its duration.  These run here as two gloo
processes.  The reference arm under torchrun: rank 0 alone works and prints.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    local_ms = 100.0 + 7.0 * rank                      # ranks finish at different times
    m = d.max(local_ms, torch.device("cpu"))
    d.barrier()
    value = bench.replica_value(d.world, tokens_per_step=4096, steps=5, ms_max=m)
    q.put((rank, m, value))
    d.done()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [107.0, 107.0]       # every rank sees the slowest rank's time
    expect = 2 * 4096 * 5 / (107.0 / 1e3)              # whole-job tokens / max time
    assert all(abs(o[2] - expect) < 1e-6 * expect for o in out)


def test_reference_arm_two_ranks_rank0_prints():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    # the keys every bench line carries
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"] == "tiny" and d["e2e"]["unit"] == d["unit"]
    assert {"value", "unit", "cores", "kind", "sample"} <= set(d["cpu_baseline"])
