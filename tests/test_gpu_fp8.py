"""GPU parity of the FP8 path against the fp64 oracle, through the C ABI.

The e4m3 quantisation (lf_quant_fp8_rows) decides each code in fp32, as the oracle's
quant_rows_e4m3_f32 does, so codes and scales must be equal bit for bit: on random rows
spanning eight orders of magnitude, all-zero rows, and the q and k of the 480p layer
workload. (Reading: the pages put FP8 with per-token activation scales on the model's
linear layers, 163.com deployment section; this path applies it to Q and K.)

The FP8 attention (lf_block_sparse_attn_fp8: e4m3 scores on kind::f8f6f4 tensor cores
times the per-token scales, bf16 softmax weights and V) is compared with the oracle's
attention over the same e4m3 q and k decoded exactly and the bf16 v (attention_fp8_qk),
on the GPU's lists, within the bf16 path's tolerances: small cases element by element
(ragged frames, frames shorter than a block, the dense first chunk, sharp softmaxes, a
forced split), and sampled plus split rows at full size.
"""
import numpy as np
import pytest
import torch

import lf_synth
import oracle

pytestmark = pytest.mark.gpu


def _quant_gpu(x):
    import block_sparse_attention_lf_b200 as L
    xd = x.cuda().contiguous()
    x8 = torch.empty(xd.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty(xd.shape[:-1], dtype=torch.float32, device="cuda")
    L.lf_quant_fp8_rows(xd, x8, sc)
    torch.cuda.synchronize()
    codes = x8.cpu().view(torch.float8_e4m3fn).double().numpy()
    return codes, sc.cpu().numpy()


@pytest.mark.parametrize("D", [64, 128])
def test_quant_rows_bit_exact_random(D):
    g = torch.Generator().manual_seed(D)
    mag = torch.exp(torch.randn(4096, 1, generator=g) * 4.0)
    x = (torch.randn(4096, D, generator=g) * mag).to(torch.bfloat16)
    x[7] = 0.0
    x[100, :] = 448.0
    codes, sc = _quant_gpu(x)
    out, osc = oracle.quant_rows_e4m3_f32(x)
    np.testing.assert_array_equal(sc, osc)
    np.testing.assert_array_equal(codes * sc.astype(np.float64)[:, None], out)


def test_quant_rows_bit_exact_layer480p():
    w = lf_synth.CONFIGS["layer480p"]
    q, k, v = lf_synth.make_qkv(w)
    for t in (q, k[:, :, : 8 * 1560]):
        t = t.contiguous()
        codes, sc = _quant_gpu(t)
        out, osc = oracle.quant_rows_e4m3_f32(t)
        np.testing.assert_array_equal(sc, osc.reshape(sc.shape))
        np.testing.assert_array_equal(codes * sc.astype(np.float64)[..., None], out.reshape(codes.shape))


def _fp8_call(shape_l, q, k, v, chunk, kf, kb, tail_pieces=0):
    """Selection on the bf16 inputs (lf_select_mask), then the e4m3 attention on the same lists."""
    import block_sparse_attention_lf_b200 as L
    call = L.HSACall(shape_l, chunk, kf, kb, tail_pieces=tail_pieces)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    call.pool(qd, kd)
    call.select()
    q8 = torch.empty(qd.shape, dtype=torch.uint8, device="cuda")
    k8 = torch.empty(kd.shape, dtype=torch.uint8, device="cuda")
    qs = torch.empty(qd.shape[:-1], dtype=torch.float32, device="cuda")
    ks = torch.empty(kd.shape[:-1], dtype=torch.float32, device="cuda")
    L.lf_quant_fp8_rows(qd, q8, qs)
    L.lf_quant_fp8_rows(kd, k8, ks)
    b = call.buf
    out = torch.full_like(b.out, float("nan"))
    L.lf_block_sparse_attn_fp8(shape_l, q8, k8, qs, ks, vd, b.block_list, b.block_count, b.list_cap, 0.0, out,
                               call.workspace, call.tail_pieces)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    assert st == 0, (st, detail)
    return dict(block_list=b.block_list.cpu().numpy(), block_count=b.block_count.cpu().numpy(),
                out=out.cpu().float().numpy().astype(np.float64), split=call.split)


FP8_SMALL = [
    # name, B, H, F, (n_sink, n_mem, n_recent, n_cur), chunk, kf, kb, kscale, tail_pieces
    ("ragged", 2, 3, 200, (1, 2, 1, 3), 2, 1, 2, 1.0, 0),
    ("frame_shorter_than_block", 1, 2, 40, (1, 3, 1, 2), 2, 2, 1, 1.0, 0),
    ("dense_first_chunk", 1, 2, 260, (0, 0, 0, 3), 1, 4, 2, 1.0, 0),
    ("sharp_softmax", 1, 2, 300, (1, 4, 1, 2), 2, 3, 3, 8.0, 0),
    ("long_lists_split", 1, 2, 1560, (1, 7, 1, 1), 2, 7, 25, 1.0, 5),
]


@pytest.mark.parametrize("case", FP8_SMALL, ids=[c[0] for c in FP8_SMALL])
def test_fp8_attention_small(case):
    """Every output row against the oracle's attention over the same e4m3 q and k (decoded
    exactly) and bf16 v, on the GPU's lists; the tolerances of the bf16 path (the remaining
    differences are fp32 score accumulation and the bf16 softmax weights, as there)."""
    import zlib
    import block_sparse_attention_lf_b200 as L
    from tests import parity
    name, B, H, F, (ns, nm, nr, nc), chunk, kf, kb, kscale, pieces = case
    NF = ns + nm + nr + nc
    g = torch.Generator().manual_seed(zlib.crc32(name.encode()) % 1000)
    q = torch.randn(B, H, nc * F, 128, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, NF * F, 128, generator=g) * kscale).to(torch.bfloat16)
    v = torch.randn(B, H, NF * F, 128, generator=g).to(torch.bfloat16)
    ls = L.LfShape.make(B, H, 128, F, NF, ns, nr, nc)
    r = _fp8_call(ls, q, k, v, chunk, kf, kb, tail_pieces=pieces)
    s = oracle.Shape(B, H, 128, F, 64, NF, ns, nr, nc)
    ref = oracle.attention_fp8_qk(s, q, k, v, r["block_list"], r["block_count"])
    got = r["out"]
    assert np.isfinite(got).all()
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= parity.OUT_MAX_ABS and rel <= parity.OUT_REL_FRO, (max_abs, rel)


@pytest.mark.parametrize("name", ["layer480p", "patterns480p"])
def test_fp8_attention_full_size(name):
    """Full size with the automatic split: sampled rows of every head and the split rows."""
    import block_sparse_attention_lf_b200 as L
    from tests import parity
    w = lf_synth.CONFIGS[name]
    q, k, v = lf_synth.make_qkv(w)
    ls = L.shape_from_workload(w)
    n_sel = L.lf_frames_selected(ls, w.chunk_index, w.topk_frames)
    kb = L.lf_blocks_for_sparsity(w.sparsity, ls.Nkv, n_sel, ls.bpf)
    r = _fp8_call(ls, q, k, v, w.chunk_index, w.topk_frames, kb)
    s = oracle.shape_of(w)
    rows = parity.sample_rows(s, per_block=2, blocks_per_head=4, seed=3)
    tail, pieces = r["split"]
    n_rows = s.batch * s.heads * s.Rq
    extra = []
    for qb in range(n_rows - tail, n_rows):
        bh, rr = divmod(qb, s.Rq)
        f, j = divmod(rr, s.bpf)
        t0 = f * s.frame_tokens + j * 64
        extra += [bh * s.Lq + t0, bh * s.Lq + min(t0 + 64, (f + 1) * s.frame_tokens) - 1]
    rows = np.union1d(rows, np.array(extra, np.int64))
    ref = oracle.attention_fp8_qk(s, q, k, v, r["block_list"], r["block_count"], rows=rows)
    got = r["out"].reshape(-1, 128)[rows]
    assert np.isfinite(r["out"]).all()
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    print(f"{name} fp8: max-abs {max_abs:.2e} rel-Frobenius {rel:.2e} over {rows.size} rows")
    assert max_abs <= parity.OUT_MAX_ABS and rel <= parity.OUT_REL_FRO, (max_abs, rel)
