"""GPU-vs-oracle comparison helpers for the HSA call (test infrastructure).

Acceptance rules (floating point decides the masks, so exactness is asked only
where the decision is clear):
  * pooled tensors: |gpu - oracle| <= POOL_ATOL * max(1, max |input|) (fp32
    sums of bf16 values against fp64);
  * masks: a top-k cut is "clear" when the k-th and (k+1)-th oracle scores
    (fp64, sorted) differ by more than TIE_REL times the largest |score| among
    that cut's candidates. Rows whose every cut is clear must match the oracle
    exactly (frames and blocks). Otherwise each GPU choice must score within
    TIE_REL of the cut, the forced frames must be present and the row must
    have the right size; the block stage is then judged on the GPU's frames;
  * attention: the oracle is run on the GPU's mask (identical to its own on
    clear rows) and the outputs must satisfy max-abs <= 3e-2 and relative
    Frobenius <= 1e-2.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

import oracle

POOL_ATOL = 2e-6
TIE_REL = 1e-4
OUT_MAX_ABS = 3e-2
OUT_REL_FRO = 1e-2


def run_gpu(shape, q, k, v, chunk: int, kf: int, kb: int, scale: float = 0.0,
            kv_stride: int = 0, tail_pieces: int = 0) -> Dict[str, np.ndarray]:
    """Run the four device steps through the C ABI; returns host copies.
    ``tail_pieces`` as in ``HSACall`` (0: the automatic split of the last wave)."""
    import block_sparse_attention_lf_b200 as L
    s = L.LfShape.make(shape.batch, shape.heads, shape.head_dim, shape.frame_tokens,
                       shape.n_frames, shape.n_sink, shape.n_recent, shape.n_cur,
                       kv_stride=kv_stride)
    call = L.HSACall(s, chunk, kf, kb, softmax_scale=scale, tail_pieces=tail_pieces)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    call(qd, kd, vd)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    assert st == 0, f"device error word {st} detail {detail:#x}"
    b = call.buf
    return dict(q_pool=b.q_pool.cpu().double().numpy(), k_pool=b.k_pool.cpu().double().numpy(),
                k_frame=b.k_frame.cpu().double().numpy(), frame_sel=b.frame_sel.cpu().numpy(),
                block_list=b.block_list.cpu().numpy(), block_count=b.block_count.cpu().numpy(),
                out=b.out.cpu().float().numpy().astype(np.float64), list_cap=b.list_cap,
                split=call.split)


def check_pool(g: dict, o: dict, q, k) -> None:
    scale = max(1.0, float(q.float().abs().max()), float(k.float().abs().max()))
    for name in ("q_pool", "k_pool", "k_frame"):
        err = np.abs(g[name] - o[name]).max()
        assert err <= POOL_ATOL * scale, f"{name}: max error {err:.3e} > {POOL_ATOL * scale:.3e}"


def _clear_cut(scores: np.ndarray, k: int) -> bool:
    """True when the top-k decision over `scores` is clear-cut."""
    n = scores.size
    if k >= n or k <= 0:
        return True
    srt = np.sort(scores)[::-1]
    scale = np.abs(scores).max()
    return (srt[k - 1] - srt[k]) > TIE_REL * scale


def _within_cut(scores: np.ndarray, chosen_idx: Sequence[int], k: int) -> bool:
    """Every chosen candidate scores at least the (k+1)-th best minus the tolerance."""
    n = scores.size
    if k >= n:
        return sorted(chosen_idx) == list(range(n))
    srt = np.sort(scores)[::-1]
    floor = srt[k] - TIE_REL * np.abs(scores).max()
    return len(set(chosen_idx)) == k and all(scores[i] >= floor for i in chosen_idx)


def check_frames(shape, chunk: int, kf: int, g: dict, o: dict) -> Dict[str, int]:
    """Frame selection under the tie rule. Returns the number of clear rows (all equal
    to the oracle's), of rows with an unclear cut ("tie") and of those that differ
    from the oracle's choice ("differ", each within the cut's tolerance)."""
    gsel, osel, fsc = g["frame_sel"], o["frame_sel"], o["frame_scores"]
    assert gsel.shape == osel.shape
    if chunk == 1:
        assert (gsel == osel).all()
        return dict(exact=gsel[..., 0].size, tie=0, differ=0)
    n_sink, n_mem = shape.n_sink, shape.n_mem
    forced = list(range(n_sink)) + list(range(shape.n_frames - shape.n_recent - shape.n_cur, shape.n_frames))
    k_eff = min(kf, n_mem)
    exact = tie = differ = 0
    for idx in np.ndindex(gsel.shape[:-1]):
        row_g, row_o = gsel[idx], osel[idx]
        if _clear_cut(fsc[idx], k_eff):
            assert (row_g == row_o).all(), f"frames differ on clear row {idx}: {row_g} vs {row_o}"
            exact += 1
            continue
        tie += 1
        if (row_g == row_o).all():
            continue
        differ += 1
        assert list(row_g) == sorted(set(row_g.tolist())), f"row {idx} not ascending/unique"
        assert set(forced) <= set(row_g.tolist())
        mem = [int(f) - n_sink for f in row_g if n_sink <= f < n_sink + n_mem]
        assert _within_cut(fsc[idx], mem, k_eff), f"frame tie row {idx}: {row_g}"
    return dict(exact=exact, tie=tie, differ=differ)


def check_blocks(shape, chunk: int, kb: int, g: dict, o_q_pool, o_k_pool) -> Dict[str, int]:
    """Block selection given the GPU's frames, under the tie rule; returns the number of
    rows equal to the oracle's ("exact") and of rows that differ at a tie ("tie")."""
    gsel = g["frame_sel"]
    lst_o, cnt_o, bsc = oracle.select_blocks(shape, chunk, kb, o_q_pool, o_k_pool, gsel,
                                             list_cap=g["list_cap"])
    glst, gcnt = g["block_list"], g["block_count"]
    assert (gcnt == cnt_o).all(), "block counts differ"
    bpf = shape.bpf
    per = bpf if chunk == 1 else min(kb, bpf)
    exact = tie = 0
    for idx in np.ndindex(gcnt.shape):
        c = int(gcnt[idx])
        row_g, row_o = glst[idx][:c], lst_o[idx][:c]
        if (row_g == row_o).all():
            exact += 1
            continue
        # differing rows must be ties in every differing frame
        tie += 1
        for s_i, tau in enumerate(gsel[idx]):
            gj = [int(b) - tau * bpf for b in row_g[s_i * per:(s_i + 1) * per]]
            oj = [int(b) - tau * bpf for b in row_o[s_i * per:(s_i + 1) * per]]
            if gj == oj:
                continue
            sc = bsc[idx + (s_i,)]
            assert not _clear_cut(sc, per), f"blocks differ on a clear cut: row {idx} frame {tau}: {gj} vs {oj}"
            assert _within_cut(sc, gj, per), f"block tie row {idx} frame {tau}: {gj}"
    return dict(exact=exact, tie=tie)


def check_attention(shape, q, k, v, g: dict, scale: Optional[float] = None,
                    rows: Optional[np.ndarray] = None) -> Dict[str, float]:
    """Oracle attention on the GPU's mask vs the GPU output (all or sampled rows)."""
    lst, cnt = g["block_list"], g["block_count"]
    out_g = g["out"].reshape(-1, shape.head_dim)
    if rows is None:
        ref = oracle.attention(shape, q, k, v, lst, cnt, scale=scale).reshape(-1, shape.head_dim)
        got = out_g
    else:
        ref = oracle.attention(shape, q, k, v, lst, cnt, scale=scale, rows=rows)
        got = out_g[rows]
    assert np.isfinite(out_g).all(), "non-finite output"
    max_abs = float(np.abs(got - ref).max())
    rel_fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= OUT_MAX_ABS, f"max-abs {max_abs:.3e}"
    assert rel_fro <= OUT_REL_FRO, f"rel-Frobenius {rel_fro:.3e}"
    return dict(max_abs=max_abs, rel_fro=rel_fro)


def sample_rows(shape, per_block: int = 3, blocks_per_head: int = 6, seed: int = 0) -> np.ndarray:
    """Flat query rows covering the first, last and partial query blocks of
    every head plus a few random ones, with first/last/random rows of each."""
    rng = np.random.default_rng(seed)
    bpf, F, Rq = shape.bpf, shape.frame_tokens, shape.Rq
    rows = []
    for bh in range(shape.batch * shape.heads):
        blocks = {0, Rq - 1, bpf - 1}
        while len(blocks) < min(Rq, blocks_per_head):
            blocks.add(int(rng.integers(0, Rq)))
        for r in sorted(blocks):
            f, j = divmod(r, bpf)
            t0 = f * F + j * 64
            n = min(64, F - j * 64)
            picks = {0, n - 1} | {int(x) for x in rng.integers(0, n, size=max(0, per_block - 2))}
            rows += [bh * shape.Lq + t0 + p for p in sorted(picks)]
    return np.array(rows, np.int64)
