"""Host logic of the multi-process benchmark path, as world-size-2 gloo ranks
on the CPU: process-group set-up from the launcher's environment, the
max-over-ranks timing reduction, and the per-rank independent workloads of
the weak-scaling run (the call shards by (batch, head) with no exchange)."""
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


def _rank_main(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), LF_DIST_BACKEND="gloo")
    import bench
    dist, r, n, local = bench._dist()
    try:
        m = bench._max_over_ranks(dist, float(10 * rank + 3))
        w = bench._rank_workload("tiny", r)
        dist.barrier()
        q.put((r, n, local, m, w.seed, w.batch, w.heads, w.n_frames))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    (r0, n0, l0, m0, s0, *shape0), (r1, n1, l1, m1, s1, *shape1) = got
    assert (r0, r1) == (0, 1) and n0 == n1 == 2 and (l0, l1) == (0, 1)
    assert m0 == m1 == 13.0            # max over ranks of 3 and 13
    assert s0 != s1                    # independent data per rank
    assert shape0 == shape1            # same per-rank work: weak scaling


def test_single_process_has_no_group(monkeypatch):
    sys.path.insert(0, ROOT)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    import bench
    dist, r, n, local = bench._dist()
    assert dist is None and (r, n, local) == (0, 1, 0)
    assert bench._max_over_ranks(None, 4.5) == 4.5
