"""The attention entry point that allocates nothing: lf_block_sparse_attn_static.

Some callers of this library cannot allocate device memory themselves: a plug-in
inside a host application that owns the whole device-memory budget and gives it
no allocator, or a loop that must not call cudaMalloc / cudaFree, which
synchronise the device and can fail once the budget is spent. For them the
attention's split of the last wave keeps its partial rows in a scratch array
compiled into the library instead of a caller workspace.

Checked here through the C ABI against the existing entry point
(lf_block_sparse_attn, whole lists, no scratch) on the same block lists, within
the output tolerance of the other parity tests: two calls in a row (the second
finds the first call's partial rows still in the array), the automatic split at
the layer480p size, forced splits of two small cases (run after the large one,
so the array holds another shape's rows), and the refusal of a split that needs
more than the array holds. The layer480p output is also compared with the fp64
oracle on sampled rows (the split rows among them), and the device's free
memory is the same before and after a call (the entry point allocates
nothing). This file is collected last.
"""
import ctypes
import os
import re
import zlib

import numpy as np
import pytest
import torch

import block_sparse_attention_lf_b200 as L
import lf_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

_P = ctypes.c_void_p
_HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lf_hsa.h")


def _scratch_bytes() -> int:
    m = re.search(r"#define LF_ATTN_STATIC_SCRATCH_BYTES \((\d+)ll << (\d+)\)", open(_HEADER).read())
    return int(m.group(1)) << int(m.group(2))


def _stream():
    return _P(torch.cuda.current_stream().cuda_stream)


def _static(shape, q, k, v, b, out, tail_pieces):
    return L.lib.lf_block_sparse_attn_static(
        ctypes.byref(shape), _P(q.data_ptr()), _P(k.data_ptr()), _P(v.data_ptr()),
        _P(b.block_list.data_ptr()), _P(b.block_count.data_ptr()), b.list_cap, 0.0,
        _P(out.data_ptr()), tail_pieces, _stream())


def _existing(shape, q, k, v, b, out):
    return L.lib.lf_block_sparse_attn(
        ctypes.byref(shape), _P(q.data_ptr()), _P(k.data_ptr()), _P(v.data_ptr()),
        _P(b.block_list.data_ptr()), _P(b.block_count.data_ptr()), b.list_cap, 0.0,
        _P(out.data_ptr()), _stream())


def _lists(shape, chunk, kf, kb, q, k):
    """Pooling and selection through the library (this test may allocate; the entry point may not)."""
    call = L.HSACall(shape, chunk, kf, kb, tail_pieces=1)
    call.pool(q, k)
    call.select()
    return call.buf


def _two_calls_match(shape, q, k, v, b, tail_pieces):
    """Two calls in a row against the existing entry point; returns the last output."""
    ref = torch.empty_like(b.out)
    assert _existing(shape, q, k, v, b, ref) == 0
    r = ref.float().cpu().numpy().astype(np.float64)
    outs = [torch.full_like(b.out, float("nan")) for _ in range(2)]  # every row must be written
    torch.cuda.synchronize()
    for i, out in enumerate(outs):
        free0 = torch.cuda.mem_get_info()[0]
        assert _static(shape, q, k, v, b, out, tail_pieces) == 0
        torch.cuda.synchronize()
        if i == 1:
            # the first call on the device may load the module; the next allocates nothing
            assert torch.cuda.mem_get_info()[0] == free0, "lf_block_sparse_attn_static changed free device memory"
        st, detail = L.lf_get_device_error()
        assert st == 0, f"device error word {st} detail {detail:#x}"
        g = out.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        assert np.abs(g - r).max() <= parity.OUT_MAX_ABS
        assert np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30) <= parity.OUT_REL_FRO
    return outs[-1]


def _layer480p(host=False):
    w = lf_synth.CONFIGS["layer480p"]
    shape = L.shape_from_workload(w)
    n_sel = L.lf_frames_selected(shape, w.chunk_index, w.topk_frames)
    kb = w.topk_blocks or L.lf_blocks_for_sparsity(w.sparsity, shape.Nkv, n_sel, shape.bpf)
    qh, kh, vh = lf_synth.make_qkv(w)
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    b = _lists(shape, w.chunk_index, w.topk_frames, kb, q, k)
    return (shape, q, k, v, b, (w, qh, kh, vh)) if host else (shape, q, k, v, b)


def test_static_scratch_layer480p_two_calls():
    shape, q, k, v, b, (w, qh, kh, vh) = _layer480p(host=True)
    tail, pieces, nbytes = L.lf_attn_split_plan(shape, b.list_cap)
    assert tail > 0 and pieces >= 2 and 0 < nbytes <= _scratch_bytes()  # the array is used
    out = _two_calls_match(shape, q, k, v, b, 0)
    # the same output against the fp64 oracle on the GPU's lists: sampled rows of every head
    # plus the first and last row of each split query block
    s_or = oracle.shape_of(w)
    rows = parity.sample_rows(s_or, per_block=2, blocks_per_head=3, seed=11)
    n_rows = shape.batch * shape.heads * shape.Rq
    split = []
    for qb in range(n_rows - tail, n_rows):
        bh, r = divmod(qb, shape.Rq)
        f, j = divmod(r, shape.bpf)
        t0 = f * shape.frame_tokens + j * 64
        split += [bh * shape.Lq + t0, bh * shape.Lq + min(t0 + 64, (f + 1) * shape.frame_tokens) - 1]
    rows = np.union1d(rows, np.array(split, np.int64))
    g = dict(block_list=b.block_list.cpu().numpy(), block_count=b.block_count.cpu().numpy(),
             out=out.float().cpu().numpy().astype(np.float64))
    parity.check_attention(s_or, qh, kh, vh, g, rows=rows)


@pytest.mark.parametrize("B,H,D,F,frames,chunk,kf,kb,pieces", [
    (2, 3, 128, 200, (1, 2, 1, 3), 2, 1, 2, 2),  # 72 query blocks x 2 pieces, ragged frames
    (1, 2, 64, 100, (1, 2, 1, 1), 2, 2, 1, 3),   # head_dim 64, lists of 5
])
def test_static_scratch_forced_split_two_calls(B, H, D, F, frames, chunk, kf, kb, pieces):
    ns, nm, nr, nc = frames
    NF = ns + nm + nr + nc
    shape = L.LfShape.make(B, H, D, F, NF, ns, nr, nc)
    g = torch.Generator().manual_seed(zlib.crc32(f"{B}{H}{D}{F}".encode()) % 1000)
    q = torch.randn(B, H, nc * F, D, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H, NF * F, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H, NF * F, D, generator=g).to(torch.bfloat16).cuda()
    b = _lists(shape, chunk, kf, kb, q, k)
    _two_calls_match(shape, q, k, v, b, pieces)


def test_static_scratch_refuses_oversize_split():
    shape, q, k, v, b = _layer480p()
    out = torch.zeros_like(b.out)
    # every list cut into list_cap pieces: far more slots than the array holds
    assert _static(shape, q, k, v, b, out, b.list_cap) == 12  # LF_ERR_SCRATCH
    torch.cuda.synchronize()
    assert int(out.view(torch.int16).abs().max()) == 0  # nothing was launched
    assert L.lib.lf_status_string(12).decode().startswith("the call needs more")
