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


def _shard_main(rank, ws, port, q):
    """One rank of a split call: its (batch, head) units through the oracle."""
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=timedelta(seconds=60))
    try:
        import block_sparse_attention_lf_b200 as L
        import lf_synth
        import oracle
        w = lf_synth.workload("tiny", batch=2, heads=3)  # 6 units: 3 + 3 over 2 ranks, 1 + 2 + 1 + 2 over 4
        q_, k_, v_ = lf_synth.make_qkv(w)
        sub, u0, u1 = L.shard_shape(L.shape_from_workload(w), ws, rank)
        ranges = [None] * ws
        dist.all_gather_object(ranges, (u0, u1))
        out = lst = cnt = None
        if sub is not None:
            qs, ks, vs = (L.unit_view(t, u0, u1).contiguous() for t in (q_, k_, v_))
            s = oracle.Shape(sub.batch, sub.heads, sub.head_dim, sub.frame_tokens, 64, sub.n_frames,
                             sub.n_sink, sub.n_recent, sub.n_cur)
            qp, kp, kf = oracle.pool(s, qs, ks)
            sel, _ = oracle.select_frames(s, w.chunk_index, w.topk_frames, qp, kf)
            lst, cnt, _ = oracle.select_blocks(s, w.chunk_index, w.topk_blocks, qp, kp, sel)
            out = oracle.attention(s, qs, ks, vs, lst, cnt)
        q.put((rank, (u0, u1), ranges, out, lst, cnt))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 4])
def test_split_call_partitions_units(ws):
    """The (batch, head) units of one call split over gloo ranks: every unit is taken by
    exactly one rank, and the ranks' outputs (the oracle on each rank's slice, a pointer
    offset into the [B, H, L, D] tensors) put back together equal the whole call."""
    import numpy as np
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=180) for _ in range(ws)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    ranges = got[0][2]
    assert all(g[2] == ranges for g in got)
    units = [u for (u0, u1) in ranges for u in range(u0, u1)]
    assert units == list(range(6))  # each unit once, in order, contiguous per rank
    sys.path.insert(0, ROOT)
    import lf_synth
    import oracle
    w = lf_synth.workload("tiny", batch=2, heads=3)
    q_, k_, v_ = lf_synth.make_qkv(w)
    s = oracle.shape_of(w)
    qp, kp, kf = oracle.pool(s, q_, k_)
    sel, _ = oracle.select_frames(s, w.chunk_index, w.topk_frames, qp, kf)
    lst, cnt, _ = oracle.select_blocks(s, w.chunk_index, w.topk_blocks, qp, kp, sel)
    out = oracle.attention(s, q_, k_, v_, lst, cnt)
    parts = [g for g in got if g[3] is not None]
    cat = lambda i: np.concatenate([g[i].reshape((-1,) + g[i].shape[2:]) for g in parts])
    np.testing.assert_array_equal(cat(3), out.reshape((-1,) + out.shape[2:]))
    np.testing.assert_array_equal(cat(4), lst.reshape((-1,) + lst.shape[2:]))
    np.testing.assert_array_equal(cat(5), cnt.reshape(-1, cnt.shape[-1]))


def test_bench_rank_inputs_strong_and_weak():
    """bench.py's per-rank inputs: strong scaling hands each rank its contiguous unit range of
    one call (the same bytes as the call's slice, idle ranks past the unit count); weak scaling
    hands every rank a whole workload's units of a call whose batch grows with the ranks."""
    sys.path.insert(0, ROOT)
    import torch
    import bench
    import block_sparse_attention_lf_b200 as L
    import lf_synth
    w = lf_synth.CONFIGS["tiny"]
    q, k, v = lf_synth.make_qkv(w)
    seen = []
    for r in range(3):  # 2 units over 3 ranks: one idle
        wr, s, qr, kr, vr, (u0, u1) = bench._rank_inputs(L, lf_synth, "tiny", r, 3, True)
        seen += list(range(u0, u1))
        if s is None:
            assert u0 == u1
            continue
        assert (s.batch, s.heads) == (1, u1 - u0)
        assert torch.equal(qr, q.reshape(-1, *q.shape[2:])[u0:u1].unsqueeze(0))
        assert torch.equal(vr, v.reshape(-1, *v.shape[2:])[u0:u1].unsqueeze(0))
    assert seen == [0, 1]
    ranges = [bench._rank_inputs(L, lf_synth, "tiny", r, 2, False)[5] for r in range(2)]
    assert ranges == [(0, 2), (2, 4)]
