"""Host logic of the benchmark's metric: the FLOPs credited to one call.

The metric counts 4 * head_dim multiply-adds-and-adds for every (query token,
kept key token) pair of the mask (the QK^T and PV products of the attention over
the kept blocks, paper.rainbus.top, execution flow, stage 3). Checked against a
count that walks query tokens one by one, on ragged frames whose last block is
partial on both the query and the key side.
"""
import numpy as np
import pytest

import bench


@pytest.mark.parametrize("F,n_cur,NF,seed", [(200, 2, 5, 0), (128, 3, 6, 1), (100, 1, 4, 2)])
def test_credited_flops_counts_mask_pairs(F, n_cur, NF, seed):
    rng = np.random.default_rng(seed)
    B, H, D, bt = 2, 3, 16, 64
    bpf = -(-F // bt)
    Rq, Nkv, Lq = n_cur * bpf, NF * bpf, n_cur * F
    cap = 5
    lst = np.full((B, H, Rq, cap), -1, np.int32)
    cnt = rng.integers(0, cap + 1, size=(B, H, Rq)).astype(np.int32)
    for idx in np.ndindex(cnt.shape):
        lst[idx][:cnt[idx]] = np.sort(rng.choice(Nkv, cnt[idx], replace=False))
    expect = 0
    for b in range(B):
        for h in range(H):
            for t in range(Lq):
                r = (t // F) * bpf + (t % F) // bt
                for g in lst[b, h, r, :cnt[b, h, r]]:
                    j = int(g) % bpf
                    expect += 4 * D * (min(F, (j + 1) * bt) - j * bt)
    assert bench.credited_flops(lst, cnt, F, bpf, D, n_cur) == float(expect)
