"""GPU parity of the whole HSA call against the fp64 oracle, through the C ABI.

Small cases are checked element by element (every pooled value, every mask row
under the tie rule, every output row); they span several tiles, ragged frames
(partial 64-token blocks), odd list lengths, frames shorter than one block, a
KV head stride larger than the used length, the dense first chunk, all-keep
masks and sharp softmaxes that force many online-softmax rescales. The five
named workloads run at full size in the launch configuration the benchmark
uses, with every mask row and pooled value checked and a sample of output rows
recomputed by the oracle.
"""
import zlib

import numpy as np
import pytest
import torch

import lf_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def _rand(seed, B, H, Lq, Lkv, D, kscale=1.0, kv_stride=0):
    g = torch.Generator().manual_seed(seed)
    Ls = kv_stride or Lkv
    q = torch.randn(B, H, Lq, D, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, Ls, D, generator=g) * kscale).to(torch.bfloat16)
    v = torch.randn(B, H, Ls, D, generator=g).to(torch.bfloat16)
    return q, k, v


def _full_check(shape, q, k, v, chunk, kf, kb, kv_stride=0, rows=None, tail_pieces=0):
    g = parity.run_gpu(shape, q, k, v, chunk, kf, kb, kv_stride=kv_stride, tail_pieces=tail_pieces)
    s_or = oracle.Shape(shape.batch, shape.heads, shape.head_dim, shape.frame_tokens, 64,
                        shape.n_frames, shape.n_sink, shape.n_recent, shape.n_cur, kv_stride=kv_stride)
    qp, kp, kfr = oracle.pool(s_or, q, k)
    sel, fsc = oracle.select_frames(s_or, chunk, kf, qp, kfr)
    o = dict(q_pool=qp, k_pool=kp, k_frame=kfr, frame_sel=sel, frame_scores=fsc)
    parity.check_pool(g, o, q, k)
    fr = parity.check_frames(s_or, chunk, kf, g, o)
    bl = parity.check_blocks(s_or, chunk, kb, g, qp, kp)
    at = parity.check_attention(s_or, q, k, v, g, rows=rows)
    return fr, bl, at


SMALL = [
    # name, B, H, D, F, (n_sink, n_mem, n_recent, n_cur), chunk, kf, kb, kscale, kv_pad
    ("ragged_d128", 2, 3, 128, 200, (1, 2, 1, 3), 2, 1, 2, 1.0, 0),
    ("ragged_d64_odd_lists", 1, 2, 64, 100, (1, 2, 1, 1), 2, 2, 1, 1.0, 0),
    ("frame_shorter_than_block", 1, 2, 128, 40, (1, 3, 1, 2), 2, 2, 1, 1.0, 0),
    ("exact_blocks", 2, 2, 128, 128, (1, 4, 1, 2), 2, 2, 1, 1.0, 0),
    ("kv_head_stride", 2, 2, 128, 150, (1, 3, 1, 2), 2, 2, 2, 1.0, 77),
    ("dense_first_chunk", 1, 2, 128, 260, (0, 0, 0, 3), 1, 4, 2, 1.0, 0),
    ("all_keep", 1, 2, 128, 190, (1, 2, 1, 2), 2, 9, 9, 1.0, 0),
    ("no_memory_frames", 1, 2, 128, 130, (1, 0, 1, 2), 2, 4, 2, 1.0, 0),
    ("no_sink_no_recent", 1, 2, 64, 256, (0, 5, 0, 2), 2, 2, 3, 1.0, 0),
    ("sharp_softmax_rescales", 1, 2, 128, 300, (1, 4, 1, 2), 2, 3, 3, 8.0, 0),
    ("long_lists_many_tiles", 1, 2, 128, 1560, (1, 7, 1, 1), 2, 7, 25, 1.0, 0),
    # fewer selected frames than the fused selection's warps: one, two and three slots
    ("single_frame_dense", 1, 2, 128, 100, (0, 0, 0, 1), 1, 1, 2, 1.0, 0),
    ("two_slots", 1, 2, 128, 150, (0, 1, 0, 1), 2, 1, 2, 1.0, 0),
    ("three_slots", 2, 2, 64, 90, (1, 1, 0, 1), 2, 1, 1, 1.0, 0),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_cases_full(case):
    name, B, H, D, F, (ns, nm, nr, nc), chunk, kf, kb, kscale, pad = case
    NF = ns + nm + nr + nc
    shape = oracle.Shape(B, H, D, F, 64, NF, ns, nr, nc)
    stride = NF * F + pad if pad else 0
    q, k, v = _rand(zlib.crc32(name.encode()) % 1000, B, H, nc * F, NF * F, D, kscale, stride)
    _full_check(shape, q, k, v, chunk, kf, kb, kv_stride=stride)


def test_tiny_workload_full():
    w = lf_synth.CONFIGS["tiny"]
    q, k, v = lf_synth.make_qkv(w)
    shape = oracle.shape_of(w)
    fr, bl, at = _full_check(shape, q, k, v, w.chunk_index, w.topk_frames, w.topk_blocks)
    assert fr["exact"] > 0


def _tail_rows(shape, chunk, kf, kb):
    """First and last valid token rows of every query block whose list the automatic plan
    splits (the last, partial wave of one-CTA-per-query-block attention)."""
    import block_sparse_attention_lf_b200 as L
    s = L.LfShape.make(shape.batch, shape.heads, shape.head_dim, shape.frame_tokens, shape.n_frames,
                       shape.n_sink, shape.n_recent, shape.n_cur)
    tail, pieces, _ = L.lf_attn_split_plan(s, L.lf_list_capacity(s, chunk, kf, kb))
    n_rows = shape.batch * shape.heads * shape.Rq
    out = []
    for qb in range(n_rows - tail, n_rows):
        bh, r = divmod(qb, shape.Rq)
        f, j = divmod(r, shape.bpf)
        t0 = f * shape.frame_tokens + j * 64
        t1 = min(t0 + 64, (f + 1) * shape.frame_tokens) - 1
        out += [bh * shape.Lq + t0, bh * shape.Lq + t1]
    return np.array(out, dtype=np.int64)


def _kb(w, shape):
    if w.topk_blocks:
        return w.topk_blocks
    n_sel = oracle.frames_selected(shape, w.chunk_index, w.topk_frames)
    return oracle.blocks_for_sparsity(w.sparsity, shape.Nkv, n_sel, shape.bpf)


def _head_rows(shape, bh):
    """Every query row of (batch*head) index bh."""
    return np.arange(bh * shape.Lq, (bh + 1) * shape.Lq, dtype=np.int64)


@pytest.mark.parametrize("name,kb_override", [("layer480p", None), ("longvideo480p", None),
                                              ("patterns480p", None), ("patterns480p", 6)])
def test_full_size_workloads(name, kb_override):
    """Full size, the benchmark's launch configuration (automatic split of the last wave).
    Every pooled value and mask row is checked; output rows: a sample of every head, the
    split query blocks' first and last rows, and at layer480p every row of the last head
    (4680 rows, which hold the split query blocks)."""
    w = lf_synth.CONFIGS[name]
    q, k, v = lf_synth.make_qkv(w)
    shape = oracle.shape_of(w)
    kb = kb_override or _kb(w, shape)
    rows = parity.sample_rows(shape, per_block=3, blocks_per_head=5, seed=1)
    rows = np.union1d(rows, _tail_rows(shape, w.chunk_index, w.topk_frames, kb))
    if name == "layer480p":
        rows = np.union1d(rows, _head_rows(shape, shape.batch * shape.heads - 1))
    fr, bl, at = _full_check(shape, q, k, v, w.chunk_index, w.topk_frames, kb, rows=rows)
    n_rows = shape.batch * shape.heads * shape.Rq
    print(f"{name} k_b {kb}: frame rows clear {fr['exact']}, unclear {fr['tie']} "
          f"(differing {fr['differ']}); block rows equal {bl['exact']}, differing at ties {bl['tie']}; "
          f"max-abs {at['max_abs']:.2e} rel-Frobenius {at['rel_fro']:.2e} over {rows.size} rows")
    # fp32 scores against fp64 ones: a choice can differ only where two candidates' scores agree
    # to about fp32 rounding, which the planted structure makes rare; a selection fault that
    # stays inside the tie tolerance on many rows fails here
    assert fr["differ"] <= max(1, n_rows // 1000)
    assert bl["tie"] <= max(1, n_rows // 1000)


def test_rollout_chunks():
    """The 7-chunk rollout: chunk 1 dense, chunks 2-7 with the Chunk-Aware Growth budgets
    computed by the library (lf_cag_budget, lf_blocks_for_sparsity), which must equal the
    oracle's."""
    import block_sparse_attention_lf_b200 as L
    w = lf_synth.CONFIGS["rollout480p"]
    qa, ka, va = lf_synth.make_rollout_qkv(w)
    n_chunks = int(w.extra["n_chunks"])
    T = list(range(1, n_chunks + 1))
    st, s_lib, beta_lib = L.lf_cag_budget(T, T, w.extra["s_base"], w.sparsity, True)
    rc, s, beta = oracle.cag(np.arange(1, n_chunks + 1), np.arange(1, n_chunks + 1),
                             w.extra["s_base"], w.sparsity, True)
    assert st == 0 and rc == 0
    assert abs(beta_lib - beta) <= 1e-12 and np.allclose(s_lib, s, rtol=0, atol=1e-12)
    for chunk in range(1, n_chunks + 1):
        wc, q, k, v = lf_synth.rollout_chunk(w, qa, ka, va, chunk)
        shape = oracle.shape_of(wc)
        ls = L.shape_from_workload(wc)
        n_sel = L.lf_frames_selected(ls, chunk, w.topk_frames)
        assert n_sel == oracle.frames_selected(shape, chunk, w.topk_frames)
        if chunk == 1:
            kb = shape.bpf
        else:
            kb = L.lf_blocks_for_sparsity(s_lib[chunk - 1], ls.Nkv, n_sel, ls.bpf)
            assert kb == oracle.blocks_for_sparsity(s[chunk - 1], shape.Nkv, n_sel, shape.bpf)
        rows = parity.sample_rows(shape, per_block=2, blocks_per_head=3, seed=chunk)
        _full_check(shape, q, k, v, chunk, w.topk_frames, kb, rows=rows)


def test_pool_range_reuses_past_frames():
    """Pooled-key cache: after a full pooling of one chunk's keys, re-pooling only
    the current-chunk frames of new keys gives exactly the full pooling of the new
    keys (past frames untouched, same per-frame arithmetic), and both match the
    oracle."""
    import block_sparse_attention_lf_b200 as L
    w = lf_synth.CONFIGS["layer480p"]
    q, k, v = lf_synth.make_qkv(w)
    shape = oracle.shape_of(w)
    ls = L.shape_from_workload(w)
    NF, C = ls.n_frames, ls.n_cur
    k2 = k.clone()
    F = ls.frame_tokens
    g = torch.Generator().manual_seed(7)
    k2[:, :, (NF - C) * F:, :] = torch.randn(k2[:, :, (NF - C) * F:, :].shape, generator=g).to(torch.bfloat16)
    qd, kd, k2d = q.cuda(), k.cuda(), k2.cuda()
    D = ls.head_dim
    mk = lambda *s: torch.full(s, float("nan"), dtype=torch.float32, device="cuda")
    qp, kp, kfr = mk(ls.batch, ls.heads, ls.Rq, D), mk(ls.batch, ls.heads, ls.Nkv, D), mk(ls.batch, ls.heads, NF, D)
    L.lf_pool(ls, qd, kd, qp, kp, kfr)
    L.lf_pool_range(ls, qd, k2d, NF - C, NF, qp, kp, kfr, pool_q=False)
    qp2, kp2, kfr2 = mk(ls.batch, ls.heads, ls.Rq, D), mk(ls.batch, ls.heads, ls.Nkv, D), mk(ls.batch, ls.heads, NF, D)
    L.lf_pool(ls, qd, k2d, qp2, kp2, kfr2)
    torch.cuda.synchronize()
    assert torch.equal(kp, kp2) and torch.equal(kfr, kfr2) and torch.equal(qp, qp2)
    oq, ok, of = oracle.pool(shape, q, k2)
    parity.check_pool({"q_pool": qp2.cpu().numpy(), "k_pool": kp2.cpu().numpy(), "k_frame": kfr2.cpu().numpy()},
                      {"q_pool": oq, "k_pool": ok, "k_frame": of}, q, k2)
    # an empty range leaves everything as it was
    before = kp.clone()
    L.lf_pool_range(ls, qd, kd, 3, 3, qp, kp, kfr, pool_q=False)
    torch.cuda.synchronize()
    assert torch.equal(before, kp)


SPLIT = [("ragged_d128", 2), ("ragged_d64_odd_lists", 3), ("kv_head_stride", 2),
         ("all_keep", 5), ("sharp_softmax_rescales", 4), ("long_lists_many_tiles", 7),
         ("long_lists_many_tiles", 1000)]


@pytest.mark.parametrize("name,pieces", SPLIT, ids=[f"{n}-{p}" for n, p in SPLIT])
def test_small_cases_split(name, pieces):
    """Every list cut into `pieces` pieces (fewer query blocks than SMs: all of them are in the
    last wave); 1000 pieces leaves most pieces empty (the count is capped at the list length)."""
    case = next(c for c in SMALL if c[0] == name)
    _, B, H, D, F, (ns, nm, nr, nc), chunk, kf, kb, kscale, pad = case
    NF = ns + nm + nr + nc
    shape = oracle.Shape(B, H, D, F, 64, NF, ns, nr, nc)
    stride = NF * F + pad if pad else 0
    q, k, v = _rand(zlib.crc32(name.encode()) % 1000, B, H, nc * F, NF * F, D, kscale, stride)
    g = parity.run_gpu(shape, q, k, v, chunk, kf, kb, kv_stride=stride, tail_pieces=pieces)
    assert g["split"][0] == B * H * shape.Rq and g["split"][1] >= 2
    s_or = oracle.Shape(B, H, D, F, 64, NF, ns, nr, nc, kv_stride=stride)
    parity.check_attention(s_or, q, k, v, g)


def test_split_matches_unsplit_layer480p():
    """The automatic split changes only the last wave's query blocks, and those only by rounding."""
    w = lf_synth.CONFIGS["layer480p"]
    q, k, v = lf_synth.make_qkv(w)
    shape = oracle.shape_of(w)
    kb = _kb(w, shape)
    a = parity.run_gpu(shape, q, k, v, w.chunk_index, w.topk_frames, kb, tail_pieces=1)
    b = parity.run_gpu(shape, q, k, v, w.chunk_index, w.topk_frames, kb)
    tail, pieces = b["split"]
    assert a["split"] == (0, 0) and tail > 0 and pieces >= 2
    np.testing.assert_array_equal(a["block_list"], b["block_list"])
    oa, ob = a["out"].reshape(-1, shape.head_dim), b["out"].reshape(-1, shape.head_dim)
    n_rows = shape.batch * shape.heads * shape.Rq
    bh0, r0 = divmod(n_rows - tail, shape.Rq)
    f0, j0 = divmod(r0, shape.bpf)
    first_tail_row = bh0 * shape.Lq + f0 * shape.frame_tokens + j0 * 64
    np.testing.assert_array_equal(oa[:first_tail_row], ob[:first_tail_row])
    d = np.abs(oa[first_tail_row:] - ob[first_tail_row:]).max()
    assert d <= parity.OUT_MAX_ABS, d


# Shapes for the selection launch only: many memory frames (200 and 805 memory frames of
# 8 blocks; 7 and 26 frame-key slots per lane in the frame level).
LARGE_SELECTION = [
    ("200_memory_frames", 1, 1, 64, 512, (1, 200, 1, 3), 2, 8, 3, 1.0, 0),
    ("805_memory_frames", 1, 1, 64, 512, (1, 805, 1, 3), 2, 8, 3, 1.0, 0),
]


@pytest.mark.parametrize("name,chunk", [("ragged_d128", 2), ("ragged_d64_odd_lists", 2), ("dense_first_chunk", 1),
                                        ("no_memory_frames", 2), ("single_frame_dense", 1), ("two_slots", 2),
                                        ("three_slots", 2), ("layer480p", 2), ("longvideo480p", 2),
                                        ("200_memory_frames", 2), ("805_memory_frames", 2)])
def test_fused_selection_equals_two_kernels(name, chunk):
    """lf_select_mask (both levels in one launch) writes exactly what lf_select_frames followed by
    lf_select_blocks write: same frame rows, lists and counts, bit for bit."""
    import block_sparse_attention_lf_b200 as L
    if name in lf_synth.CONFIGS:
        w = lf_synth.CONFIGS[name]
        q, k, v = lf_synth.make_qkv(w)
        ls = L.shape_from_workload(w)
        kf = w.topk_frames
        n_sel = L.lf_frames_selected(ls, chunk, kf)
        kb = w.topk_blocks or L.lf_blocks_for_sparsity(w.sparsity, ls.Nkv, n_sel, ls.bpf)
    else:
        case = next(c for c in SMALL + LARGE_SELECTION if c[0] == name)
        _, B, H, D, F, (ns, nm, nr, nc), _, kf, kb, kscale, _ = case
        ls = L.LfShape.make(B, H, D, F, ns + nm + nr + nc, ns, nr, nc)
        q, k, v = _rand(zlib.crc32(name.encode()) % 1000, B, H, nc * F, ls.n_frames * F, D, kscale)
    call = L.HSACall(ls, chunk, kf, kb)
    b = call.buf
    call.pool(q.cuda(), k.cuda())
    fs2, bl2, bc2 = torch.full_like(b.frame_sel, -5), torch.full_like(b.block_list, -5), torch.full_like(b.block_count, -5)
    L.lf_select_frames(ls, chunk, kf, b.q_pool, b.k_frame, fs2)
    L.lf_select_blocks(ls, chunk, kf, kb, b.q_pool, b.k_pool, fs2, bl2, bc2, b.list_cap)
    b.frame_sel.fill_(-9)
    b.block_list.fill_(-9)
    b.block_count.fill_(-9)
    call.select()
    torch.cuda.synchronize()
    assert L.lf_get_device_error()[0] == 0
    assert torch.equal(b.frame_sel, fs2) and torch.equal(b.block_count, bc2)
    cnt = int(bc2.max())
    assert torch.equal(b.block_list[..., :cnt], bl2[..., :cnt])


def test_dependent_launches_see_their_producers():
    """The selection and the attention are launched as programmatic dependents of the kernel
    before them and wait for it before reading. Back-to-back calls with no host
    synchronisation, each preceded by a torch kernel that rewrites q, k and v, must give
    every call the output of its own inputs: the output of each call equals the output of
    the same inputs run alone (bit for bit, the same kernels)."""
    import block_sparse_attention_lf_b200 as L
    w = lf_synth.CONFIGS["layer480p"]
    shape = L.shape_from_workload(w)
    n_sel = L.lf_frames_selected(shape, w.chunk_index, w.topk_frames)
    kb = w.topk_blocks or L.lf_blocks_for_sparsity(w.sparsity, shape.Nkv, n_sel, shape.bpf)
    q0, k0, v0 = (t.cuda() for t in lf_synth.make_qkv(w))
    call = L.HSACall(shape, w.chunk_index, w.topk_frames, kb)
    scales = (1.0, -0.5, 2.0)
    alone = []
    for sc in scales:
        call(q0 * sc, k0 * sc, v0 * sc)
        torch.cuda.synchronize()
        alone.append(call.buf.out.clone())
    q, k, v = torch.empty_like(q0), torch.empty_like(k0), torch.empty_like(v0)
    chained = []
    for sc in scales:
        torch.mul(q0, sc, out=q)
        torch.mul(k0, sc, out=k)
        torch.mul(v0, sc, out=v)
        call(q, k, v)
        chained.append(call.buf.out.clone())  # a torch kernel after the attention's merge
    torch.cuda.synchronize()
    assert L.lf_get_device_error()[0] == 0
    for a, c in zip(alone, chained):
        assert torch.equal(a, c)
