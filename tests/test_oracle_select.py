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
