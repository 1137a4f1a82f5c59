"""Pins for the oracle's block-sparse softmax attention.

Source: Light Forcing (paper.rainbus.top), execution flow, stage 3 (block-sparse
attention over the mask B_r). The pages fix no scale and no causal mask; the
readings used are scale = 1/sqrt(D), softmax over exactly the valid tokens of
the kept blocks, and no causal mask inside the current chunk.

Pins: (1) when the selection keeps every frame and block the result must be
dense softmax attention, computed here by torch's fp64 scaled-dot-product
attention (a library routine); (2) one kept block equals softmax over that
block's tokens, written out with numpy; (3) an explicit token set that includes
a partial block excludes the positions past the frame's end; (4) every output
is a convex combination of the kept values.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand_bf16(g, *shape, scale=1.0):
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("F,bt,D", [(100, 64, 16), (64, 64, 8), (40, 64, 8), (130, 64, 32)])
def test_all_keep_equals_dense_sdpa(F, bt, D):
    g = torch.Generator().manual_seed(F + D)
    B, H, NF, n_cur = 2, 2, 5, 2
    s = oracle.Shape(B, H, D, F, bt, NF, 1, 1, n_cur)
    q = _rand_bf16(g, B, H, s.Lq, D)
    k = _rand_bf16(g, B, H, s.Lkv, D, scale=2.0)
    v = _rand_bf16(g, B, H, s.Lkv, D)
    # k_f >= |M| and k_b >= bpf keep everything
    res = oracle.run_hsa(s, q, k, v, chunk_index=2, topk_frames=99, topk_blocks=99)
    assert (res["block_count"] == s.Nkv).all()
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-12)
    # the dense first chunk takes the same path regardless of k
    res1 = oracle.run_hsa(s, q, k, v, chunk_index=1, topk_frames=1, topk_blocks=1)
    np.testing.assert_allclose(res1["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_single_block_and_partial_block():
    g = torch.Generator().manual_seed(3)
    B, H, D, F, bt, NF, n_cur = 1, 1, 8, 100, 64, 3, 1
    s = oracle.Shape(B, H, D, F, bt, NF, 0, 0, n_cur)
    q = _rand_bf16(g, B, H, s.Lq, D)
    k = _rand_bf16(g, B, H, s.Lkv, D, scale=3.0)
    v = _rand_bf16(g, B, H, s.Lkv, D)
    bpf = s.bpf  # 2: tokens 0-63 and 64-99
    scale = 0.37
    qd, kd, vd = q.double().numpy()[0, 0], k.double().numpy()[0, 0], v.double().numpy()[0, 0]
    for g_blk in [0, 1, 3, 5]:  # full and partial blocks of frames 0, 1, 2
        lst = np.full((B, H, s.Rq, 1), g_blk, np.int32)
        cnt = np.ones((B, H, s.Rq), np.int32)
        out = oracle.attention(s, q, k, v, lst, cnt, scale=scale)[0, 0]
        tau, j = divmod(g_blk, bpf)
        toks = np.arange(tau * F + j * bt, tau * F + min((j + 1) * bt, F))
        z = scale * qd @ kd[toks].T
        p = np.exp(z - z.max(1, keepdims=True))
        ref = (p / p.sum(1, keepdims=True)) @ vd[toks]
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # two blocks: partial block 1 of frame 0 plus full block 0 of frame 2
    lst = np.array([1, 4], np.int32).reshape(1, 1, 1, 2).repeat(s.Rq, 2)
    cnt = np.full((B, H, s.Rq), 2, np.int32)
    out = oracle.attention(s, q, k, v, lst, cnt, scale=scale)[0, 0]
    toks = np.concatenate([np.arange(64, 100), np.arange(200, 264)])
    z = scale * qd @ kd[toks].T
    p = np.exp(z - z.max(1, keepdims=True))
    ref = (p / p.sum(1, keepdims=True)) @ vd[toks]
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_rows_subset_and_empty_list():
    """Computing a subset of rows gives the same numbers as the full call; a
    row with an empty block list returns zeros (a reading: softmax over an
    empty set is undefined)."""
    g = torch.Generator().manual_seed(5)
    s = oracle.Shape(2, 3, 16, 70, 64, 4, 1, 1, 1)
    q = _rand_bf16(g, 2, 3, s.Lq, 16)
    k = _rand_bf16(g, 2, 3, s.Lkv, 16)
    v = _rand_bf16(g, 2, 3, s.Lkv, 16)
    res = oracle.run_hsa(s, q, k, v, 2, 1, 1)
    full = res["out"].reshape(-1, 16)
    rows = [0, 5, 69, 70, 139, 300, 2 * 3 * 70 - 1]
    part = oracle.attention(s, q, k, v, res["block_list"], res["block_count"], rows=rows)
    np.testing.assert_array_equal(part, full[rows])
    cnt = res["block_count"].copy()
    cnt[1, 2, 0] = 0
    out = oracle.attention(s, q, k, v, res["block_list"], cnt)
    assert (out[1, 2, :64] == 0).all()


def test_value_is_convex_combination():
    """Each output coordinate lies between the min and max of the kept values."""
    g = torch.Generator().manual_seed(9)
    s = oracle.Shape(1, 2, 8, 100, 64, 6, 1, 1, 2)
    q = _rand_bf16(g, 1, 2, s.Lq, 8)
    k = _rand_bf16(g, 1, 2, s.Lkv, 8, scale=4.0)
    v = _rand_bf16(g, 1, 2, s.Lkv, 8)
    res = oracle.run_hsa(s, q, k, v, 2, 2, 1)
    vd = v.double().numpy()
    assert np.all(res["out"] <= vd.max(axis=2, keepdims=True) + 1e-12)
    assert np.all(res["out"] >= vd.min(axis=2, keepdims=True) - 1e-12)


def test_per_query_block_lists():
    """Every query block gets its own two-block list; each query row is checked
    against softmax over the tokens of its own block's list, with the query
    block found from (frame, block-in-frame) as the pages' block mask is
    indexed per query block of the current chunk."""
    g = torch.Generator().manual_seed(21)
    B, H, D, F, bt, NF, n_cur = 1, 2, 8, 100, 64, 4, 2
    s = oracle.Shape(B, H, D, F, bt, NF, 1, 0, n_cur)
    q = _rand_bf16(g, B, H, s.Lq, D)
    k = _rand_bf16(g, B, H, s.Lkv, D, scale=2.0)
    v = _rand_bf16(g, B, H, s.Lkv, D)
    lst = np.zeros((B, H, s.Rq, 2), np.int32)
    for h in range(H):
        for r in range(s.Rq):
            a = (3 * r + h) % s.Nkv
            b = (a + 1 + (5 * r + h) % (s.Nkv - 1)) % s.Nkv  # never equal to a
            lst[0, h, r] = sorted((a, b))
    cnt = np.full((B, H, s.Rq), 2, np.int32)
    out = oracle.attention(s, q, k, v, lst, cnt)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for h in range(H):
        for t in range(s.Lq):
            f, j = divmod(t, F)
            r = f * s.bpf + j // bt
            toks = []
            for gb in lst[0, h, r]:
                tau, jj = divmod(int(gb), s.bpf)
                toks += list(range(tau * F + jj * bt, tau * F + min((jj + 1) * bt, F)))
            z = qd[0, h, t] @ kd[0, h, toks].T / np.sqrt(D)
            p = np.exp(z - z.max())
            np.testing.assert_allclose(out[0, h, t], (p / p.sum()) @ vd[0, h, toks], rtol=1e-12, atol=1e-13)
