"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The step has no exchange, so N GPUs run N independent replicas; bench.py
times each on its device and reports the units of all ranks over the slowest
rank's time (max over ranks through one all-reduce). This checks that logic
with world_size 2 over gloo, and that the reference arm prints only on rank 0.
"""

import io
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

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

    dist = bench.init_dist(world, "gloo")
    try:
        m = bench.max_over_ranks(1.5 * (rank + 1), dist)
        bench.barrier(dist)
        value, ms = bench.aggregate_throughput(100, 10.0 * (rank + 1), dist)
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"])
        q.put((rank, m, value, ms, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_and_reference_arm():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, m, value, ms, out in res:
        assert m == 3.0
        assert ms == 20.0
        assert abs(value - 200 / 0.020) < 1e-6
        lines = [ln for ln in out.splitlines() if ln.startswith("{")]
        assert len(lines) == (1 if rank == 0 else 0)
    import json

    rec = json.loads([ln for ln in res[0][4].splitlines() if ln.startswith("{")][0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
