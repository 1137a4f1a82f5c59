"""The C-ABI library loads, exports what include/lf_hsa.h declares, and its host
logic (CAG solver, block-count mapping, sizes, argument validation) matches the
oracle. No CUDA device is touched: every device entry point called here fails
validation before it could launch anything."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_lf_b200 as L
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lf_hsa.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^LF_API\s+[\w\s\*]+?\b(lf_\w+)\(", txt, re.M)))


def test_exports_match_header():
    declared = _declared()
    assert declared == sorted(L.ABI_FUNCTIONS)
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    exported = sorted(m.group(1) for m in re.finditer(r" T (lf_\w+)$", out, re.M))
    assert exported == declared
    for name in declared:
        assert hasattr(L.lib, name)


def test_shape_struct_layout():
    # 9 int32 fields, 4 bytes of padding, one int64
    assert ctypes.sizeof(L.LfShape) == 48
    assert L.LfShape.kv_stride.offset == 40


def test_version():
    assert "sm_100a" in L.lf_version()


@pytest.mark.parametrize("seed", range(30))
def test_cag_matches_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 10))
    T = np.cumsum(rng.uniform(0.2, 3.0, n))
    w = rng.uniform(0.1, 4.0, n) if seed % 3 else None
    s_base = rng.uniform(0.6, 0.99)
    s_target = rng.uniform(0.05, 0.95) * s_base
    over_all = bool(seed % 2)
    st, s, beta = L.lf_cag_budget(list(T), None if w is None else list(w), s_base, s_target, over_all)
    rc, so, bo = oracle.cag(T, w, s_base, s_target, over_all)
    assert (st == 0) == (rc == 0)
    if st in (0, 6):  # values are reported for feasible and infeasible budgets
        assert beta == pytest.approx(bo, rel=1e-12, abs=1e-15)
        np.testing.assert_allclose(s, so, rtol=1e-12, atol=1e-15)


def test_cag_errors():
    assert L.lf_cag_budget([1.0], None, 0.9, 0.5)[0] == 9                 # one chunk
    assert L.lf_cag_budget([1.0, 0.0], None, 0.9, 0.5)[0] == 9            # T <= 0
    assert L.lf_cag_budget([1.0, 2.0], [1.0, -1.0], 0.9, 0.5)[0] == 9     # w <= 0
    assert L.lf_cag_budget([1.0, 2.0], None, 1.2, 0.5)[0] == 9            # s_base outside [0,1)
    assert L.lf_cag_budget([1.0, 2.0, 3.0], None, 0.5, 0.6)[0] == 6       # beta < 0
    assert L.lib.lf_cag_budget(3, None, None, 0.9, 0.5, 1, None, None) == 1


def test_cag_rollout_default_matches_oracle():
    st, s, beta = L.lf_cag_budget(list(range(1, 8)), None, 0.95, 0.80, True)
    rc, so, bo = oracle.cag(np.arange(1, 8), np.arange(1, 8), 0.95, 0.80, True)
    assert st == 0 and rc == 0
    assert beta == pytest.approx(bo, rel=1e-14)
    np.testing.assert_allclose(s, so, rtol=1e-14)


@pytest.mark.parametrize("s", [0.0, 0.3, 0.5, 0.79, 0.8, 0.81, 0.9, 0.95, 0.999])
@pytest.mark.parametrize("nkv,nsel,bpf", [(525, 9, 25), (1625, 9, 25), (36, 6, 4), (75, 6, 25)])
def test_blocks_for_sparsity_matches_oracle(s, nkv, nsel, bpf):
    assert L.lf_blocks_for_sparsity(s, nkv, nsel, bpf) == oracle.blocks_for_sparsity(s, nkv, nsel, bpf)


def test_sizes_match_oracle():
    for (NF, ns, nr, nc) in [(21, 1, 1, 3), (9, 1, 1, 2), (3, 0, 0, 3), (65, 1, 1, 3), (5, 2, 0, 3)]:
        sh = L.LfShape.make(1, 2, 128, 1560, NF, ns, nr, nc)
        os_ = oracle.Shape(1, 2, 128, 1560, 64, NF, ns, nr, nc)
        for chunk in (1, 2, 5):
            for kf in (1, 4, 100):
                n = L.lf_frames_selected(sh, chunk, kf)
                assert n == oracle.frames_selected(os_, chunk, kf)
                for kb in (1, 12, 25, 40):
                    per = 25 if chunk == 1 else min(kb, 25)
                    assert L.lf_list_capacity(sh, chunk, kf, kb) == n * per


def _shape(**kw):
    base = dict(batch=1, heads=2, head_dim=128, frame_tokens=1560, n_frames=21, n_sink=1,
                n_recent=1, n_cur=3)
    base.update(kw)
    return L.LfShape.make(**base)


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=96), 3), (dict(block_tokens=32), 3), (dict(frame_tokens=0), 3),
    (dict(frame_tokens=9000), 3), (dict(n_cur=0), 3), (dict(n_frames=4), 3),
    (dict(n_sink=-1), 3), (dict(batch=0), 3), (dict(kv_stride=100), 3),
    (dict(n_frames=1030, n_sink=1, n_recent=1, n_cur=3), 3),
])
def test_shape_validation(bad, code):
    sh = _shape(**bad)
    p = ctypes.c_void_p(FAKE)
    assert L.lib.lf_pool(ctypes.byref(sh), p, p, p, p, p, None) == code
    assert L.lib.lf_select_frames(ctypes.byref(sh), 2, 4, p, p, p, None) == code
    assert L.lib.lf_select_blocks(ctypes.byref(sh), 2, 4, 12, p, p, p, p, p, 1000, None) == code
    assert L.lib.lf_block_sparse_attn(ctypes.byref(sh), p, p, p, p, p, 1000, 0.0, p, None) == code
    assert L.lib.lf_select_blocks_1d(ctypes.byref(sh), 2, 12, p, p, p, p, 1000, None) == code
    assert L.lf_frames_selected(sh, 2, 4) == -1
    assert L.lf_list_capacity(sh, 2, 4, 12) == -1


def test_argument_validation():
    sh = _shape()
    p = ctypes.c_void_p(FAKE)
    mis = ctypes.c_void_p(FAKE + 8)
    S = ctypes.byref(sh)
    assert L.lib.lf_pool(None, p, p, p, p, p, None) == 1
    assert L.lib.lf_pool(S, None, p, p, p, p, None) == 1
    assert L.lib.lf_pool(S, p, mis, p, p, p, None) == 2
    assert L.lib.lf_select_frames(S, 0, 4, p, p, p, None) == 9      # chunk index is 1-based
    assert L.lib.lf_select_frames(S, 2, 0, p, p, p, None) == 4      # top-k below 1
    assert L.lib.lf_select_frames(S, 2, 4, p, None, p, None) == 1
    assert L.lib.lf_select_frames(S, 2, 4, p, p, mis, None) == 2
    assert L.lib.lf_select_blocks(S, 2, 4, 0, p, p, p, p, p, 108, None) == 4
    assert L.lib.lf_select_blocks(S, 2, 4, 12, p, p, p, p, p, 107, None) == 5   # cap < 9*12
    assert L.lib.lf_select_blocks(S, 2, 4, 12, p, p, p, None, p, 108, None) == 1
    assert L.lib.lf_block_sparse_attn(S, p, p, p, p, p, -1, 0.0, p, None) == 5
    assert L.lib.lf_block_sparse_attn(S, p, p, p, p, p, 108, float("nan"), p, None) == 9
    assert L.lib.lf_block_sparse_attn(S, p, p, None, p, p, 108, 0.0, p, None) == 1
    assert L.lib.lf_block_sparse_attn(S, p, p, p, p, p, 108, 0.0, mis, None) == 2


def test_pool_range_validation():
    sh = _shape()
    p = ctypes.c_void_p(FAKE)
    mis = ctypes.c_void_p(FAKE + 8)
    S = ctypes.byref(sh)
    nf = sh.n_frames
    f = L.lib.lf_pool_range
    assert f(S, p, p, -1, nf, 1, p, p, p, None) == 9          # frame_begin < 0
    assert f(S, p, p, 3, 2, 1, p, p, p, None) == 9            # begin > end
    assert f(S, p, p, 0, nf + 1, 1, p, p, p, None) == 9       # end past the last frame
    assert f(S, None, p, 0, nf, 1, p, p, p, None) == 1        # q needed when pooling q
    assert f(S, p, p, 0, nf, 1, None, p, p, None) == 1
    assert f(S, None, p, 0, nf, 0, None, p, None, None) == 1   # k_frame always needed
    assert f(S, None, mis, nf - 3, nf, 0, None, p, p, None) == 2  # q may be NULL without pool_q
    assert f(None, p, p, 0, 1, 1, p, p, p, None) == 1
    bad = _shape(head_dim=96)
    assert f(ctypes.byref(bad), p, p, 0, 1, 1, p, p, p, None) == 3


def test_status_strings():
    for code in range(12):
        assert L.lf_status_string(code)
    assert L.lf_status_string(99) == "unknown status"


def test_binding_rejects_cpu_tensors():
    import torch
    sh = _shape(heads=1, n_frames=5, n_sink=1, n_recent=1, n_cur=1, frame_tokens=64)
    q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        L.lf_pool(sh, q, q, q.float(), q.float(), q.float())


def test_attn_ws_validation():
    sh = _shape()
    p = ctypes.c_void_p(FAKE)
    mis = ctypes.c_void_p(FAKE + 8)
    S = ctypes.byref(sh)
    f = L.lib.lf_block_sparse_attn_ws
    assert f(ctypes.byref(_shape(head_dim=96)), p, p, p, p, p, 108, 0.0, p, 0, p, 1 << 20, None) == 3
    assert f(S, p, p, p, p, p, -1, 0.0, p, 0, p, 1 << 20, None) == 5
    assert f(S, p, p, p, p, p, 108, 0.0, p, -1, p, 1 << 20, None) == 9   # tail_pieces < 0
    assert f(S, p, p, p, p, p, 108, 0.0, p, 0, p, -16, None) == 9        # workspace_bytes < 0
    assert f(S, p, p, p, p, p, 108, 0.0, p, 0, None, 1 << 20, None) == 1  # bytes without a workspace
    assert f(S, p, p, p, p, p, 108, 0.0, p, 0, mis, 1 << 20, None) == 2
    assert f(S, p, p, None, p, p, 108, 0.0, p, 0, p, 1 << 20, None) == 1


def _plan_rule(n_rows, sm, cap):
    """The split rule as the header states it."""
    r = n_rows % sm
    if r == 0 or sm // r < 8:
        return 0, 0
    k = min(sm // r, cap // 8, cap)
    return (r, k) if k >= 2 else (0, 0)


@pytest.mark.parametrize("B,H,nc,kb,sm", [
    (1, 12, 3, 12, 148),   # 900 query blocks: 12 in the last wave, lists of 108
    (2, 12, 3, 12, 148),   # 1800: 24 in the last wave
    (1, 2, 3, 12, 148),    # 150: 2 left over
    (1, 1, 1, 12, 148),    # fewer query blocks than SMs: every list split
    (1, 12, 3, 1, 148),    # lists of 9 entries: pieces capped at 9 // 8 = 1, no split
    (1, 4, 37, 12, 148),   # 4 * 37 * 25 = 3700 = 25 waves of 148: no tail
    (1, 12, 3, 12, 132),   # another SM count
    (1, 24, 3, 12, 148),   # 1800 = 12 waves + 24: the last wave fills 16 % of the SMs, no split
])
def test_split_plan(B, H, nc, kb, sm):
    sh = L.LfShape.make(B, H, 128, 1560, 18 + nc, 1, 1, nc)
    cap = L.lf_list_capacity(sh, 2, 4, kb)
    t, k, nbytes = L.lf_attn_split_plan(sh, cap, sm)
    n_rows = B * H * sh.Rq
    assert (t, k) == _plan_rule(n_rows, sm, cap)
    assert nbytes == t * k * 64 * (128 + 2) * 4
    if (B, H, nc, kb, sm) == (1, 12, 3, 12, 148):
        assert (t, k) == (12, 12)


def test_split_plan_validation():
    sh = _shape()
    t, k, b = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int64()
    f = L.lib.lf_attn_split_plan
    assert f(ctypes.byref(sh), -1, 148, ctypes.byref(t), ctypes.byref(k), ctypes.byref(b)) == 5
    assert f(ctypes.byref(sh), 108, 148, None, ctypes.byref(k), ctypes.byref(b)) == 1
    assert f(ctypes.byref(_shape(head_dim=96)), 108, 148, ctypes.byref(t), ctypes.byref(k), ctypes.byref(b)) == 3


def test_select_1d_validation():
    sh = _shape()  # 21 frames x 25 blocks = 525 candidates
    p = ctypes.c_void_p(FAKE)
    mis = ctypes.c_void_p(FAKE + 8)
    S = ctypes.byref(sh)
    f = L.lib.lf_select_blocks_1d
    assert f(S, 0, 12, p, p, p, p, 108, None) == 9      # chunk index is 1-based
    assert f(S, 2, 0, p, p, p, p, 108, None) == 4       # top-k below 1
    assert f(S, 2, 108, None, p, p, p, 108, None) == 1
    assert f(S, 2, 108, p, mis, p, p, 108, None) == 2
    assert f(S, 2, 108, p, p, p, p, 107, None) == 5     # list shorter than the kept count
    assert f(S, 1, 1, p, p, p, p, 524, None) == 5       # chunk 1 keeps all 525
    assert f(S, 2, 10 ** 6, p, p, p, p, 524, None) == 5  # k above Nkv keeps all 525
    big = _shape(n_frames=700, n_sink=1, n_recent=1, n_cur=3)  # 17500 candidates
    assert f(ctypes.byref(big), 2, 12, p, p, p, p, 100, None) == 3


def test_frame_index_validation():
    """lf_frame_index_build / lf_select_frames_ivf reject bad arguments before launching."""
    import ctypes
    s = L.LfShape.make(1, 2, 128, 1560, 21, 1, 1, 3)
    P = ctypes.c_void_p
    p16 = P(4096)
    ok_ptrs = [p16] * 5
    # n_clusters outside 1..64, negative iters
    assert L.lib.lf_frame_index_build(ctypes.byref(s), 0, 5, *ok_ptrs, None) == 9
    assert L.lib.lf_frame_index_build(ctypes.byref(s), 65, 5, *ok_ptrs, None) == 9
    assert L.lib.lf_frame_index_build(ctypes.byref(s), 8, -1, *ok_ptrs, None) == 9
    assert L.lib.lf_frame_index_build(ctypes.byref(s), 8, 5, p16, None, p16, p16, p16, None) == 1
    assert L.lib.lf_frame_index_build(ctypes.byref(s), 8, 5, P(4100), p16, p16, p16, p16, None) == 2
    bad = L.LfShape.make(1, 2, 96, 1560, 21, 1, 1, 3)
    assert L.lib.lf_frame_index_build(ctypes.byref(bad), 8, 5, *ok_ptrs, None) == 3
    sel_ptrs = [p16] * 6
    assert L.lib.lf_select_frames_ivf(ctypes.byref(s), 2, 4, 8, 0, *sel_ptrs, None) == 9   # n_probe < 1
    assert L.lib.lf_select_frames_ivf(ctypes.byref(s), 0, 4, 8, 2, *sel_ptrs, None) == 9   # chunk < 1
    assert L.lib.lf_select_frames_ivf(ctypes.byref(s), 2, 0, 8, 2, *sel_ptrs, None) == 4   # top-k < 1
    assert L.lib.lf_select_frames_ivf(ctypes.byref(s), 2, 4, 8, 2, p16, p16, p16, p16, p16, None, None) == 1
