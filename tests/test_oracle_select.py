"""Pins for the oracle's two-level mask selection.

Source: Light Forcing (paper.rainbus.top), execution flow, stage 3 (frame top-k
with the sink, most recent and current-chunk frames always kept; block top-k
inside each selected frame; mask B_r(tau,j) = 1[tau in T_r, j in J_r(tau)]);
gist.science Technical Summary 2.2 (two-level mask selection, attention cost
independent of the number of history frames). Ties go to the lower index (a
reading; the pages are silent).
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _topk_by_definition(scores, k):
    """The unique k-subset S with: for i in S, j not in S, s_i > s_j or
    (s_i == s_j and i < j). Found by enumerating every k-subset."""
    n = len(scores)
    k = min(k, n)
    found = []
    for S in itertools.combinations(range(n), k):
        Sset = set(S)
        ok = all(scores[i] > scores[j] or (scores[i] == scores[j] and i < j)
                 for i in S for j in range(n) if j not in Sset)
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def test_select_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "topk_hand.json")))
    NF, bpf = g["n_frames"], g["bpf"]
    s = oracle.Shape(1, 1, 2, bpf * 64, 64, NF, g["n_sink"], g["n_recent"], g["n_cur"])
    assert s.bpf == bpf
    Rq = s.Rq
    q_pool = np.tile(np.array(g["q_pool"], np.float64), (1, 1, Rq, 1)).reshape(1, 1, Rq, 2)
    k_frame = np.zeros((1, 1, NF, 2))
    k_frame[0, 0, :, 0] = g["frame_first_coord"]
    k_frame[0, 0, :, 1] = 5.0  # orthogonal to q~, must not matter
    k_pool = np.zeros((1, 1, NF * bpf, 2))
    for tau in range(NF):
        k_pool[0, 0, tau * bpf:(tau + 1) * bpf, 0] = g["block_first_coord"]
        k_pool[0, 0, tau * bpf:(tau + 1) * bpf, 1] = -3.0
    for kf, expect in g["expect_frames"].items():
        sel, _ = oracle.select_frames(s, 2, int(kf), q_pool, k_frame)
        for r in range(Rq):
            assert sel[0, 0, r].tolist() == expect
    sel, _ = oracle.select_frames(s, 2, 2, q_pool, k_frame)
    for kb, in_frame in g["expect_blocks_in_frame"].items():
        lst, cnt, _ = oracle.select_blocks(s, 2, int(kb), q_pool, k_pool, sel)
        expect = [tau * bpf + j for tau in g["expect_frames"]["2"] for j in in_frame]
        for r in range(Rq):
            assert cnt[0, 0, r] == len(expect)
            assert lst[0, 0, r, :cnt[0, 0, r]].tolist() == expect


@pytest.mark.parametrize("seed", range(6))
def test_select_brute_force_with_ties(seed):
    """Integer-valued pooled vectors give many exact ties; compare both levels
    against the subset-enumeration definition of top-k."""
    rng = np.random.default_rng(seed)
    B, H, D, bt = 1, 2, 3, 64
    NF, n_sink, n_recent, n_cur = 9, 1, 1, 2
    bpf = 5
    s = oracle.Shape(B, H, D, bpf * bt - 10, bt, NF, n_sink, n_recent, n_cur)
    Rq = s.Rq
    q_pool = rng.integers(-2, 3, size=(B, H, Rq, D)).astype(np.float64)
    k_frame = rng.integers(-2, 3, size=(B, H, NF, D)).astype(np.float64)
    k_pool = rng.integers(-2, 3, size=(B, H, NF * bpf, D)).astype(np.float64)
    kf, kb = 1 + seed % 4, 1 + seed % 5
    sel, fsc = oracle.select_frames(s, 2, kf, q_pool, k_frame)
    lst, cnt, _ = oracle.select_blocks(s, 2, kb, q_pool, k_pool, sel)
    mem = list(range(n_sink, NF - n_recent - n_cur))
    for b in range(B):
        for h in range(H):
            for r in range(Rq):
                scores = [float(q_pool[b, h, r] @ k_frame[b, h, m]) for m in mem]
                np.testing.assert_array_equal(fsc[b, h, r], scores)
                top = [mem[i] for i in _topk_by_definition(scores, kf)]
                expect_T = sorted(list(range(n_sink)) + top + list(range(NF - n_recent - n_cur, NF)))
                assert sel[b, h, r].tolist() == expect_T
                expect_list = []
                for tau in expect_T:
                    bs = [float(q_pool[b, h, r] @ k_pool[b, h, tau * bpf + j]) for j in range(bpf)]
                    expect_list += [tau * bpf + j for j in _topk_by_definition(bs, kb)]
                assert cnt[b, h, r] == len(expect_list)
                assert lst[b, h, r, :cnt[b, h, r]].tolist() == sorted(expect_list)


@pytest.mark.parametrize("chunk_index,kf,kb", [(2, 2, 2), (2, 9, 3), (2, 1, 99), (1, 2, 2)])
def test_select_invariants(chunk_index, kf, kb):
    """Forced frames always present; |T_r| = n_sink + min(k_f,|M|) + n_recent +
    n_cur; each row keeps exactly |T_r| * min(k_b, bpf) blocks (fixed attention
    cost); lists ascending and unique; chunk 1 keeps everything."""
    rng = np.random.default_rng(11)
    B, H, D = 2, 2, 8
    s = oracle.Shape(B, H, D, 200, 64, 10, 2, 1, 2)
    q_pool = rng.standard_normal((B, H, s.Rq, D))
    k_frame = rng.standard_normal((B, H, s.n_frames, D))
    k_pool = rng.standard_normal((B, H, s.Nkv, D))
    sel, _ = oracle.select_frames(s, chunk_index, kf, q_pool, k_frame)
    lst, cnt, _ = oracle.select_blocks(s, chunk_index, kb, q_pool, k_pool, sel)
    forced = set(range(s.n_sink)) | set(range(s.n_frames - s.n_recent - s.n_cur, s.n_frames))
    n_sel = s.n_frames if chunk_index == 1 else s.n_sink + min(kf, s.n_mem) + s.n_recent + s.n_cur
    per_frame = s.bpf if chunk_index == 1 else min(kb, s.bpf)
    assert sel.shape[-1] == n_sel
    for row in sel.reshape(-1, n_sel):
        assert forced <= set(row.tolist())
        assert list(row) == sorted(set(row.tolist()))
    assert (cnt == n_sel * per_frame).all()
    for r_sel, r_lst, c in zip(sel.reshape(-1, n_sel), lst.reshape(-1, lst.shape[-1]), cnt.reshape(-1)):
        blocks = r_lst[:c].tolist()
        assert blocks == sorted(set(blocks))
        assert {g // s.bpf for g in blocks} == set(r_sel.tolist())
    if chunk_index == 1:
        assert (lst == np.arange(s.Nkv)).all()


# ---- one-dimensional selection (the ablation's single-granularity variant) ----------
# 163.com article, section 4 (ablation: one-dimensional sparse attention, no frame
# level). Reading: a global top-k over all KV blocks, no forced frames, ties to the
# lower index, ascending ids; the first chunk stays dense.

@pytest.mark.parametrize("seed", range(6))
def test_select_1d_brute_force_with_ties(seed):
    """Integer pooled vectors (many exact ties) against the subset-enumeration top-k over
    every KV block of every frame."""
    rng = np.random.default_rng(100 + seed)
    B, H, D = 1, 2, 3
    s = oracle.Shape(B, H, D, 150, 64, 4, 1, 1, 1)  # 4 frames x 3 blocks = 12 candidates
    q_pool = rng.integers(-2, 3, size=(B, H, s.Rq, D)).astype(np.float64)
    k_pool = rng.integers(-2, 3, size=(B, H, s.Nkv, D)).astype(np.float64)
    kb = 1 + seed
    lst, cnt, sc = oracle.select_blocks_1d(s, 2, kb, q_pool, k_pool)
    for b in range(B):
        for h in range(H):
            for r in range(s.Rq):
                scores = [float(q_pool[b, h, r] @ k_pool[b, h, g]) for g in range(s.Nkv)]
                np.testing.assert_array_equal(sc[b, h, r], scores)
                expect = sorted(_topk_by_definition(scores, kb))
                assert cnt[b, h, r] == len(expect)
                assert lst[b, h, r, :cnt[b, h, r]].tolist() == expect


@pytest.mark.parametrize("chunk_index,kb", [(2, 1), (2, 7), (2, 10**6), (1, 3)])
def test_select_1d_invariants(chunk_index, kb):
    """Every row keeps min(k, Nkv) blocks (all of them in the dense first chunk), as an
    ascending list of distinct valid ids; no frame is forced in."""
    rng = np.random.default_rng(12)
    B, H, D = 2, 2, 8
    s = oracle.Shape(B, H, D, 200, 64, 10, 2, 1, 2)
    q_pool = rng.standard_normal((B, H, s.Rq, D))
    k_pool = rng.standard_normal((B, H, s.Nkv, D))
    lst, cnt, _ = oracle.select_blocks_1d(s, chunk_index, kb, q_pool, k_pool)
    keep = s.Nkv if chunk_index == 1 else min(kb, s.Nkv)
    assert (cnt == keep).all()
    for r_lst, c in zip(lst.reshape(-1, lst.shape[-1]), cnt.reshape(-1)):
        blocks = r_lst[:c].tolist()
        assert blocks == sorted(set(blocks)) and 0 <= blocks[0] and blocks[-1] < s.Nkv
    if chunk_index == 1:
        assert (lst == np.arange(s.Nkv)).all()


def test_select_1d_forces_no_frame():
    """Sink blocks that score below every other block are never kept by the one-dimensional
    selection, while the two-level selection always keeps the sink frame."""
    rng = np.random.default_rng(14)
    B, H, D = 1, 2, 4
    s = oracle.Shape(B, H, D, 200, 64, 8, 1, 1, 2)
    q_pool = np.abs(rng.standard_normal((B, H, s.Rq, D))) + 0.1
    k_pool = np.abs(rng.standard_normal((B, H, s.Nkv, D))) + 0.1
    k_pool[:, :, :s.bpf * s.n_sink] = -1.0  # every sink block scores below zero
    lst, cnt, _ = oracle.select_blocks_1d(s, 2, s.Nkv - s.bpf * s.n_sink, q_pool, k_pool)
    assert (lst >= s.bpf * s.n_sink).all()
    k_frame = np.abs(rng.standard_normal((B, H, s.n_frames, D)))
    sel, _ = oracle.select_frames(s, 2, 1, q_pool, k_frame)
    assert (sel[..., 0] == 0).all()


def test_select_1d_matches_two_level_on_frame_structured_scores():
    """When every frame holds exactly k_b blocks that outscore every other block of every
    frame, the global top-(frames * k_b) is the two-level selection with all frames kept and
    top-k_b blocks per frame."""
    rng = np.random.default_rng(13)
    B, H, D, kb = 1, 2, 4, 2
    s = oracle.Shape(B, H, D, 300, 64, 6, 1, 1, 1)  # bpf 5, 3 memory frames
    q_pool = np.zeros((B, H, s.Rq, D))
    q_pool[..., 0] = 1.0
    k_pool = rng.standard_normal((B, H, s.Nkv, D)) * 0.1
    k_frame = rng.standard_normal((B, H, s.n_frames, D))
    for h in range(H):
        for tau in range(s.n_frames):
            hi = rng.choice(s.bpf, kb, replace=False)
            k_pool[0, h, tau * s.bpf + hi, 0] += 10.0 + rng.random(kb)
    sel, _ = oracle.select_frames(s, 2, s.n_mem, q_pool, k_frame)  # every frame kept
    lst2, cnt2, _ = oracle.select_blocks(s, 2, kb, q_pool, k_pool, sel)
    lst1, cnt1, _ = oracle.select_blocks_1d(s, 2, s.n_frames * kb, q_pool, k_pool)
    np.testing.assert_array_equal(cnt1, cnt2)
    np.testing.assert_array_equal(lst1, lst2)
