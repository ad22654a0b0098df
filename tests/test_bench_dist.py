"""Multi-process host logic of bench.py on CPU (gloo, world size 2):
process-group setup from the torchrun environment, the barrier, the
max-over-ranks timing reduction, and the reference arm printing on rank 0 only
while the other ranks exit 0 without work."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout
from types import SimpleNamespace

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    args = SimpleNamespace(gpus=world, steps=2, warmup=1, workload="c3", cpu_seconds=0.1)
    w, r, _ = bench.dist_setup(args)
    assert dist.get_backend() == "gloo"
    m = bench.max_over_ranks(w, 10.0 * (r + 1), torch.device("cpu"))
    bench.barrier(w)
    calls = []

    class FakeSample:
        def __init__(self, cid, seconds=15.0):
            calls.append(("init", cid))

        def run(self):
            calls.append("run")
            return {"value": 1.5e-3, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                    "sample": "fake", "sample_seconds": 0.0, "est_step_seconds": 1.0}

    bench.OracleSample = FakeSample
    out = io.StringIO()
    with redirect_stdout(out):
        rc = bench.run_reference(args, w, r)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, m, rc, out.getvalue(), calls.count("run")))


def test_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, m, rc, out, ncalls = q.get(timeout=120)
        res[r] = (m, rc, out, ncalls)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # max over ranks: both ranks see the slowest rank's value
    assert res[0][0] == res[1][0] == 20.0
    # reference arm: rank 0 prints one JSON line, rank 1 does no work
    assert res[0][1] == 0 and res[1][1] == 0
    assert res[1][2] == "" and res[1][3] == 0
    line = json.loads(res[0][2].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert res[0][3] == 3          # warmup 1 + steps 2
