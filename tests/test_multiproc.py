"""The N > 1 path of bench.py on CPU: two gloo ranks.

The decode step is independent per (sequence, KV head), so N GPUs run N
replicas with no data-path collective; what remains to check is the rank
plumbing: environment, process-group set-up, the barrier, the max over
ranks that the reported time uses, and that only rank 0 runs and prints the
reference arm.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    try:
        r, w, local = bench.dist_env()
        bench.dist_init(w, "gloo")
        bench.barrier(w)
        got = bench.max_over_ranks(float(10 + 5 * r), w)  # ranks time 10 and 15
        # the reference arm runs on rank 0 only; other ranks leave without work
        args = bench.parse(["--impl", "reference", "--gpus", str(w), "--steps", "1",
                            "--warmup", "0", "--workload", "tiny_k4v4_4k"])
        rc = 0 if r == 0 else bench.run_reference(args, bench.workload_of(args))
        bench.barrier(w)
        q.put((r, w, local, got, rc))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[2] == r[0] for r in res)
    assert all(r[3] == 15.0 for r in res)  # both ranks see the slowest rank's time
    assert res[1][4] == 0                   # rank 1 exits the reference arm cleanly
