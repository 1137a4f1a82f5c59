"""Pins for the oracle's coarse frame retrieval (an index over the frame means).

Source: Light Forcing (paper.rainbus.top), weaknesses paragraph: the frame
candidate set grows linearly with the video, and a hierarchical index is the
remedy it names; execution flow, stage 3 for the frame selection it
approximates. Reading (the pages do not fix the index): k-means with squared L2
distance over each head's memory-frame means, started at evenly spaced memory
frames; a query block probes clusters by <q~_r, centroid> until at least
n_probe clusters and k candidate frames, then takes the exact top-k of those
frames; the sink, recent and current frames stay forced.
"""
import itertools
import warnings

import numpy as np
import pytest

import oracle


def _topk_by_definition(scores, idx, k):
    """k-subset of `idx` with every member outscoring every non-member (ties: lower id)."""
    n = len(idx)
    k = min(k, n)
    found = []
    for S in itertools.combinations(range(n), k):
        Sset = set(S)
        if all(scores[i] > scores[j] or (scores[i] == scores[j] and idx[i] < idx[j])
               for i in S for j in range(n) if j not in Sset):
            found.append(sorted(idx[i] for i in S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed,C,kf", [(0, 4, 3), (1, 1, 2), (2, 7, 5), (3, 10, 1)])
def test_ivf_full_probe_equals_exact_selection(seed, C, kf):
    rng = np.random.default_rng(seed)
    s = oracle.Shape(2, 2, 8, 200, 64, 14, 1, 1, 2)  # 10 memory frames
    q_pool = rng.standard_normal((2, 2, s.Rq, 8))
    k_frame = rng.standard_normal((2, 2, s.n_frames, 8))
    exact, _ = oracle.select_frames(s, 2, kf, q_pool, k_frame)
    ivf, _, _ = oracle.select_frames_ivf(s, 2, kf, C, C, 25, q_pool, k_frame)
    np.testing.assert_array_equal(ivf, exact)


@pytest.mark.parametrize("seed", range(4))
def test_ivf_kmeans_matches_sklearn(seed):
    """Centroids and labels equal scikit-learn's Lloyd k-means run from the same initial
    centroids (memory frames floor(i*|M|/C)) for the same number of rounds."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(20 + seed)
    D, n_mem, C, iters = 6, 40, 4, 3 + seed
    s = oracle.Shape(1, 1, D, 128, 64, n_mem + 4, 1, 1, 2)
    centers = rng.standard_normal((C, D)) * 2.0
    k_frame = np.zeros((1, 1, s.n_frames, D))
    k_frame[0, 0] = rng.standard_normal((s.n_frames, D))
    k_frame[0, 0, 1:1 + n_mem] += centers[rng.integers(0, C, n_mem)]
    q_pool = rng.standard_normal((1, 1, s.Rq, D))
    _, cent, lab = oracle.select_frames_ivf(s, 2, 3, C, 1, iters, q_pool, k_frame)
    km = k_frame[0, 0, 1:1 + n_mem]
    init = km[[i * n_mem // C for i in range(C)]]
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        ref = KMeans(n_clusters=C, init=init, n_init=1, max_iter=iters, tol=0.0, algorithm="lloyd").fit(km)
    assert len(set(ref.labels_.tolist())) == C  # no empty cluster (the two handle those differently)
    np.testing.assert_array_equal(lab[0, 0], ref.labels_)
    np.testing.assert_allclose(cent[0, 0], ref.cluster_centers_, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed,C,n_probe,kf", [(0, 5, 1, 2), (1, 5, 2, 6), (2, 8, 3, 4), (3, 3, 1, 9)])
def test_ivf_probing_invariants(seed, C, n_probe, kf):
    """Row size fixed; forced frames present; the chosen memory frames lie in the probed
    clusters (the best n_probe by centroid score, extended in score order until they hold
    min(k,|M|) frames) and are the exact top-k of those clusters' frames."""
    rng = np.random.default_rng(40 + seed)
    B, H, D = 1, 2, 5
    s = oracle.Shape(B, H, D, 200, 64, 16, 1, 1, 2)  # 12 memory frames
    q_pool = rng.integers(-2, 3, size=(B, H, s.Rq, D)).astype(np.float64)
    k_frame = rng.standard_normal((B, H, s.n_frames, D))
    sel, cent, lab = oracle.select_frames_ivf(s, 2, kf, C, n_probe, 10, q_pool, k_frame)
    n_mem = s.n_mem
    k_eff = min(kf, n_mem)
    forced = set(range(s.n_sink)) | set(range(s.n_frames - s.n_recent - s.n_cur, s.n_frames))
    assert sel.shape[-1] == s.n_sink + k_eff + s.n_recent + s.n_cur
    for b in range(B):
        for h in range(H):
            for r in range(s.Rq):
                row = sel[b, h, r].tolist()
                assert row == sorted(set(row)) and forced <= set(row)
                cs = [float(q_pool[b, h, r] @ cent[b, h, j]) for j in range(cent.shape[2])]
                order = sorted(range(len(cs)), key=lambda j: (-cs[j], j))
                probed, have = [], 0
                for t, j in enumerate(order):
                    if t >= n_probe and have >= k_eff:
                        break
                    probed.append(j)
                    have += int((lab[b, h] == j).sum())
                members = [s.n_sink + m for m in range(n_mem) if lab[b, h, m] in probed]
                scores = [float(q_pool[b, h, r] @ k_frame[b, h, f]) for f in members]
                chosen = sorted(set(row) - forced)
                assert chosen == _topk_by_definition(scores, members, k_eff)


def test_ivf_dense_first_chunk():
    rng = np.random.default_rng(7)
    s = oracle.Shape(1, 1, 4, 128, 64, 9, 1, 1, 2)
    sel, _, _ = oracle.select_frames_ivf(s, 1, 2, 3, 1, 5, rng.standard_normal((1, 1, s.Rq, 4)),
                                         rng.standard_normal((1, 1, 9, 4)))
    assert (sel == np.arange(9)).all()
