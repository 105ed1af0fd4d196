"""The N > 1 host logic of bench.py on CPU: two gloo ranks in spawned processes.

Every (batch, head) pair is an independent problem, so the multi-GPU bench runs one replica
per rank with no collective on the data path; the only cross-rank steps are the barriers
around the timed region and the reduction of the device times (max over ranks) and of the
work done (sum over ranks).  The reference arm runs on rank 0 only.
"""
import contextlib
import io
import json
import os
import socket
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
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks(1.5 * (rank + 1), world)
        sm = bench.sum_over_ranks(float(rank + 1), world)
        bench.barrier(world)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "1", "--ref-pairs", "1"])
        out.put((rank, mx, sm, rc, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_reference_arm_on_rank0_only():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, mx, sm, rc, text = q.get(timeout=240)
        results[rank] = (mx, sm, rc, text)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (mx, sm, rc, text) in results.items():
        assert mx == pytest.approx(3.0)  # max over ranks of 1.5 * (rank + 1)
        assert sm == pytest.approx(3.0)  # 1 + 2
        assert rc == 0
    line = json.loads(results[0][3].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert results[1][3].strip() == ""
