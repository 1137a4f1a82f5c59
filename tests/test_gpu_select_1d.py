"""GPU parity of the one-dimensional (single-granularity) block selection, and of
the attention over its lists, against the fp64 oracle, through the C ABI.

163.com article ("南洋理工大学打造视频生成新引擎"), section 4: the ablation's
one-dimensional sparse attention has no frame level. Reading: every KV block of
the call is a candidate, o_r(g) = <q~_r, k~_g>, the row keeps the top-k with no
frame forced in, ties to the lower index, ascending ids; the first chunk is
dense. Lists are judged under the same tie rule as the two-level selection
(clear cuts exact, others within the cut tolerance); the attention over the
GPU's lists against the oracle within the usual output tolerance.
"""
import zlib

import numpy as np
import pytest
import torch

import block_sparse_attention_lf_b200 as L
import lf_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def _run_and_check(shape, q, k, v, chunk, kb, rows=None):
    s = L.LfShape.make(shape.batch, shape.heads, shape.head_dim, shape.frame_tokens, shape.n_frames,
                       shape.n_sink, shape.n_recent, shape.n_cur)
    call = L.HSACall(s, chunk, 1, 1)  # pooled buffers and the output; the selection is replaced
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    call.pool(qd, kd)
    keep = s.Nkv if (chunk == 1 or kb >= s.Nkv) else kb
    bl = torch.full((s.batch, s.heads, s.Rq, keep), -7, dtype=torch.int32, device="cuda")
    bc = torch.zeros(s.batch, s.heads, s.Rq, dtype=torch.int32, device="cuda")
    L.lf_select_blocks_1d(s, chunk, kb, call.buf.q_pool, call.buf.k_pool, bl, bc, keep)
    out = torch.empty_like(call.buf.out)
    L.lf_block_sparse_attn(s, qd, kd, vd, bl, bc, keep, 0.0, out)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    assert st == 0, f"device error word {st} detail {detail:#x}"
    g = dict(block_list=bl.cpu().numpy(), block_count=bc.cpu().numpy(),
             out=out.cpu().float().numpy().astype(np.float64), list_cap=keep)
    qp, kp, _ = oracle.pool(shape, q, k)
    lst_o, cnt_o, sc = oracle.select_blocks_1d(shape, chunk, kb, qp, kp)
    np.testing.assert_array_equal(g["block_count"], cnt_o)
    exact = tie = 0
    for idx in np.ndindex(cnt_o.shape):
        c = int(cnt_o[idx])
        row_g, row_o = g["block_list"][idx][:c], lst_o[idx][:c]
        assert list(row_g) == sorted(set(row_g.tolist())), f"row {idx} not ascending and unique"
        if (row_g == row_o).all():
            exact += 1
            continue
        tie += 1
        assert not parity._clear_cut(sc[idx], c), f"lists differ on a clear cut: row {idx}"
        assert parity._within_cut(sc[idx], [int(x) for x in row_g], c), f"tie row {idx}"
    parity.check_attention(shape, q, k, v, g, rows=rows)
    return exact, tie


def _rand(seed, B, H, Lq, Lkv, D):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, Lq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, H, Lkv, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, H, Lkv, D, generator=gen).to(torch.bfloat16)
    return q, k, v


CASES = [
    # name, B, H, D, F, (n_sink, n_mem, n_recent, n_cur), chunk, k
    ("ragged_d128", 2, 3, 128, 200, (1, 2, 1, 3), 2, 7),
    ("d64_short_list", 1, 2, 64, 100, (1, 2, 1, 1), 2, 3),
    ("dense_first_chunk", 1, 2, 128, 260, (0, 0, 0, 3), 1, 4),
    ("keep_everything", 1, 2, 128, 190, (1, 2, 1, 2), 2, 10 ** 6),
    ("525_candidates", 1, 1, 128, 1560, (1, 16, 1, 3), 2, 108),
    # many candidates per row (1,600 and 6,480 KV blocks of 8 per frame)
    ("1600_candidates", 1, 1, 64, 512, (1, 195, 1, 3), 2, 40),
    ("6480_candidates", 1, 1, 64, 512, (1, 805, 1, 3), 2, 50),
    # 32 heads x 5 tiles of 8 query blocks: more tiles than SMs (the 8-warp ring)
    ("160_tiles", 4, 8, 64, 256, (1, 3, 1, 10), 2, 9),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_select_1d_small(case):
    name, B, H, D, F, (ns, nm, nr, nc), chunk, kb = case
    NF = ns + nm + nr + nc
    shape = oracle.Shape(B, H, D, F, 64, NF, ns, nr, nc)
    q, k, v = _rand(zlib.crc32(name.encode()) % 1000, B, H, nc * F, NF * F, D)
    rows = parity.sample_rows(shape, per_block=3, blocks_per_head=4, seed=3) if F * nc * B * H > 2000 else None
    _run_and_check(shape, q, k, v, chunk, kb, rows=rows)


def test_select_1d_layer480p():
    """The 480p layer call with the same kept-block budget as the two-level selection
    (4 memory frames + 5 forced frames, 12 blocks each: 108 of 525 blocks)."""
    w = lf_synth.CONFIGS["layer480p"]
    q, k, v = lf_synth.make_qkv(w)
    shape = oracle.shape_of(w)
    n_sel = oracle.frames_selected(shape, w.chunk_index, w.topk_frames)
    kb2 = oracle.blocks_for_sparsity(w.sparsity, shape.Nkv, n_sel, shape.bpf)
    rows = parity.sample_rows(shape, per_block=2, blocks_per_head=4, seed=5)
    exact, tie = _run_and_check(shape, q, k, v, w.chunk_index, n_sel * kb2, rows=rows)
    assert exact >= 0.5 * (exact + tie)
