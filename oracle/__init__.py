"""fp64 CPU oracle for the Light Forcing HSA call (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The product path (the CUDA library and its binding)
never does, and this package never imports the product.

The arithmetic lives in ``lf_oracle.c`` (plain single-threaded C, fp64); this
module only marshals numpy arrays into it. Parity status of each routine is
listed in the header of ``lf_oracle.c``; every routine is pinned by tests in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblf_oracle.so")
_lib = None

_i = ctypes.c_int
_l = ctypes.c_long
_d = ctypes.c_double
_p = ctypes.c_void_p


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build
        _build.build()
    _lib = configure(ctypes.CDLL(_LIB_PATH))
    return _lib


def configure(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    lib.orc_pool.argtypes = [_i] * 7 + [_l, _p, _p, _p, _p, _p]
    lib.orc_pool.restype = None
    lib.orc_frames_selected.argtypes = [_i] * 6
    lib.orc_frames_selected.restype = _i
    lib.orc_select_frames.argtypes = [_i] * 10 + [_p, _p, _p, _p]
    lib.orc_select_frames.restype = None
    lib.orc_select_blocks.argtypes = [_i] * 9 + [_p, _p, _p, _p, _p, _i, _p]
    lib.orc_select_blocks.restype = _i
    lib.orc_select_frames_ivf.argtypes = [_i] * 13 + [_p, _p, _p, _p, _p]
    lib.orc_select_frames_ivf.restype = None
    lib.orc_select_blocks_1d.argtypes = [_i] * 7 + [_p, _p, _p, _p, _i, _p]
    lib.orc_select_blocks_1d.restype = _i
    lib.orc_attention.argtypes = [_i] * 6 + [_l, _p, _p, _p, _p, _p, _i, _d, _p, _l, _p]
    lib.orc_attention.restype = None
    lib.orc_e4m3.argtypes = [_d]
    lib.orc_e4m3.restype = _d
    lib.orc_e4m3_array.argtypes = [_p, _l, _p]
    lib.orc_e4m3_array.restype = None
    lib.orc_quant_rows_e4m3.argtypes = [_p, _l, _i, _p, _p]
    lib.orc_quant_rows_e4m3.restype = None
    lib.orc_quant_rows_e4m3_f32.argtypes = [_p, _l, _i, _p, _p]
    lib.orc_quant_rows_e4m3_f32.restype = None
    lib.orc_quant_cols_e4m3.argtypes = [_p, _l, _l, _l, _i, _p, _p]
    lib.orc_quant_cols_e4m3.restype = None
    lib.orc_attention_f64.argtypes = [_i] * 6 + [_l, _p, _p, _p, _p, _p, _i, _d, _p, _l, _p]
    lib.orc_attention_f64.restype = None
    lib.orc_cag.argtypes = [_i, _p, _p, _d, _d, _i, _p, _p]
    lib.orc_cag.restype = _i
    lib.orc_blocks_for_sparsity.argtypes = [_d, _i, _i, _i]
    lib.orc_blocks_for_sparsity.restype = _i
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_p)


def _bf16_bits(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 bit patterns."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


@dataclass(frozen=True)
class Shape:
    """HSA call sizes: frames are [sink..., memory..., recent..., current...]."""

    batch: int
    heads: int
    head_dim: int
    frame_tokens: int
    block_tokens: int
    n_frames: int
    n_sink: int
    n_recent: int
    n_cur: int
    kv_stride: int = 0  # tokens between consecutive heads in k/v; 0 = n_frames*frame_tokens

    @property
    def bpf(self) -> int:
        return -(-self.frame_tokens // self.block_tokens)

    @property
    def n_mem(self) -> int:
        return self.n_frames - self.n_sink - self.n_recent - self.n_cur

    @property
    def Lq(self) -> int:
        return self.n_cur * self.frame_tokens

    @property
    def Lkv(self) -> int:
        return self.n_frames * self.frame_tokens

    @property
    def Rq(self) -> int:
        return self.n_cur * self.bpf

    @property
    def Nkv(self) -> int:
        return self.n_frames * self.bpf

    @property
    def stride(self) -> int:
        return self.kv_stride or self.Lkv


def shape_of(w) -> Shape:
    """Shape from an ``lf_synth.Workload``."""
    return Shape(w.batch, w.heads, w.head_dim, w.frame_tokens, w.block_tokens,
                 w.n_frames, w.n_sink, w.n_recent, w.n_cur)


def pool(s: Shape, q, k) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Block means of q and k and frame means of k, fp64."""
    lib = _load()
    qb, kb = _bf16_bits(q), _bf16_bits(k)
    BH = s.batch * s.heads
    q_pool = np.zeros((BH * s.Rq, s.head_dim), np.float64)
    k_pool = np.zeros((BH * s.Nkv, s.head_dim), np.float64)
    k_frame = np.zeros((BH * s.n_frames, s.head_dim), np.float64)
    lib.orc_pool(s.batch, s.heads, s.head_dim, s.frame_tokens, s.block_tokens, s.n_frames,
                 s.n_cur, s.stride, _ptr(qb), _ptr(kb), _ptr(q_pool), _ptr(k_pool), _ptr(k_frame))
    return (q_pool.reshape(s.batch, s.heads, s.Rq, s.head_dim),
            k_pool.reshape(s.batch, s.heads, s.Nkv, s.head_dim),
            k_frame.reshape(s.batch, s.heads, s.n_frames, s.head_dim))


def frames_selected(s: Shape, chunk_index: int, topk_frames: int) -> int:
    return _load().orc_frames_selected(s.n_frames, s.n_sink, s.n_recent, s.n_cur,
                                       chunk_index, topk_frames)


def select_frames(s: Shape, chunk_index: int, topk_frames: int, q_pool: np.ndarray,
                  k_frame: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """T_r per (b,h,r) as [B,H,Rq,n_sel] int32, plus the memory-frame scores."""
    lib = _load()
    n_sel = frames_selected(s, chunk_index, topk_frames)
    qp = np.ascontiguousarray(q_pool, np.float64)
    kf = np.ascontiguousarray(k_frame, np.float64)
    sel = np.zeros((s.batch, s.heads, s.Rq, n_sel), np.int32)
    scores = np.zeros((s.batch, s.heads, s.Rq, max(s.n_mem, 0)), np.float64)
    lib.orc_select_frames(s.batch, s.heads, s.head_dim, s.Rq, s.n_frames, s.n_sink, s.n_recent,
                          s.n_cur, chunk_index, topk_frames, _ptr(qp), _ptr(kf), _ptr(sel),
                          _ptr(scores) if scores.size else None)
    return sel, scores


def select_blocks(s: Shape, chunk_index: int, topk_blocks: int, q_pool: np.ndarray,
                  k_pool: np.ndarray, frame_sel: np.ndarray, list_cap: Optional[int] = None
                  ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(block_list [B,H,Rq,cap], block_count [B,H,Rq], block scores [B,H,Rq,n_sel,bpf])."""
    lib = _load()
    n_sel = frame_sel.shape[-1]
    kb = s.bpf if (chunk_index == 1 or topk_blocks > s.bpf) else topk_blocks
    cap = list_cap if list_cap is not None else n_sel * kb
    qp = np.ascontiguousarray(q_pool, np.float64)
    kp = np.ascontiguousarray(k_pool, np.float64)
    fs = np.ascontiguousarray(frame_sel, np.int32)
    lst = np.full((s.batch, s.heads, s.Rq, cap), -1, np.int32)
    cnt = np.zeros((s.batch, s.heads, s.Rq), np.int32)
    sc = np.zeros((s.batch, s.heads, s.Rq, n_sel, s.bpf), np.float64)
    rc = lib.orc_select_blocks(s.batch, s.heads, s.head_dim, s.Rq, s.n_frames, s.bpf, n_sel,
                               chunk_index, topk_blocks, _ptr(qp), _ptr(kp), _ptr(fs), _ptr(lst),
                               _ptr(cnt), cap, _ptr(sc))
    if rc != 0:
        raise ValueError("block list exceeds list_cap")
    return lst, cnt, sc


def select_frames_ivf(s: Shape, chunk_index: int, topk_frames: int, n_clusters: int, n_probe: int,
                      iters: int, q_pool: np.ndarray, k_frame: np.ndarray
                      ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Frame selection through a k-means index over the memory-frame means:
    (T_r [B,H,Rq,n_sel] int32, centroids [B,H,C,D], labels [B,H,n_mem])."""
    lib = _load()
    n_sel = frames_selected(s, chunk_index, topk_frames)
    C = max(1, min(n_clusters, s.n_mem))
    qp = np.ascontiguousarray(q_pool, np.float64)
    kf = np.ascontiguousarray(k_frame, np.float64)
    sel = np.zeros((s.batch, s.heads, s.Rq, n_sel), np.int32)
    cent = np.zeros((s.batch, s.heads, C, s.head_dim), np.float64)
    lab = np.zeros((s.batch, s.heads, max(s.n_mem, 0)), np.int32)
    lib.orc_select_frames_ivf(s.batch, s.heads, s.head_dim, s.Rq, s.n_frames, s.n_sink, s.n_recent,
                              s.n_cur, chunk_index, topk_frames, n_clusters, n_probe, iters, _ptr(qp),
                              _ptr(kf), _ptr(sel), _ptr(cent), _ptr(lab) if lab.size else None)
    return sel, cent, lab


def select_blocks_1d(s: Shape, chunk_index: int, topk_blocks: int, q_pool: np.ndarray,
                     k_pool: np.ndarray, list_cap: Optional[int] = None
                     ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One-dimensional selection (global block top-k, no frame level):
    (block_list [B,H,Rq,cap], block_count [B,H,Rq], block scores [B,H,Rq,Nkv])."""
    lib = _load()
    keep = s.Nkv if (chunk_index == 1 or topk_blocks > s.Nkv) else topk_blocks
    cap = list_cap if list_cap is not None else keep
    qp = np.ascontiguousarray(q_pool, np.float64)
    kp = np.ascontiguousarray(k_pool, np.float64)
    lst = np.full((s.batch, s.heads, s.Rq, cap), -1, np.int32)
    cnt = np.zeros((s.batch, s.heads, s.Rq), np.int32)
    sc = np.zeros((s.batch, s.heads, s.Rq, s.Nkv), np.float64)
    rc = lib.orc_select_blocks_1d(s.batch, s.heads, s.head_dim, s.Rq, s.Nkv, chunk_index, topk_blocks,
                                  _ptr(qp), _ptr(kp), _ptr(lst), _ptr(cnt), cap, _ptr(sc))
    if rc != 0:
        raise ValueError("block list exceeds list_cap")
    return lst, cnt, sc


def attention(s: Shape, q, k, v, block_list: np.ndarray, block_count: np.ndarray,
              scale: Optional[float] = None, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Masked softmax attention, fp64, for flat query rows (bh*Lq + t).

    Returns [n_rows, D]; with rows=None every query row, as [B,H,Lq,D].
    """
    lib = _load()
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    lst = np.ascontiguousarray(block_list, np.int32)
    cnt = np.ascontiguousarray(block_count, np.int32)
    cap = lst.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(s.head_dim)
    full = rows is None
    if full:
        rows = np.arange(s.batch * s.heads * s.Lq, dtype=np.int64)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((r.size, s.head_dim), np.float64)
    lib.orc_attention(s.batch, s.heads, s.head_dim, s.frame_tokens, s.block_tokens, s.n_cur,
                      s.stride, _ptr(qb), _ptr(kb), _ptr(vb), _ptr(lst), _ptr(cnt), cap,
                      float(scale), _ptr(r), r.size, _ptr(out))
    if full:
        return out.reshape(s.batch, s.heads, s.Lq, s.head_dim)
    return out


def e4m3(x) -> np.ndarray:
    """Nearest e4m3 value of each element (ties to even, saturating at 448), fp64."""
    xa = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.zeros_like(xa)
    _load().orc_e4m3_array(_ptr(xa), xa.size, _ptr(out))
    return out


def quant_rows_e4m3(x) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row (per token) e4m3 quantisation of bf16 x [..., D]: (dequantised fp64, scales [...])."""
    xb = _bf16_bits(x)
    D = xb.shape[-1]
    n = xb.size // D
    out = np.zeros(xb.shape, np.float64)
    sc = np.zeros(xb.shape[:-1], np.float64)
    _load().orc_quant_rows_e4m3(_ptr(xb), n, D, _ptr(out), _ptr(sc))
    return out, sc


def quant_rows_e4m3_f32(x) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation decided in fp32 (scale fl32(amax/448), code of
    fl32(x/scale)): (dequantised fp64 [..., D], fp32 scales [...])."""
    xb = _bf16_bits(x)
    D = xb.shape[-1]
    n = xb.size // D
    out = np.zeros(xb.shape, np.float64)
    sc = np.zeros(xb.shape[:-1], np.float32)
    _load().orc_quant_rows_e4m3_f32(_ptr(xb), n, D, _ptr(out), _ptr(sc))
    return out, sc


def attention_fp8_qk(s: Shape, q, k, v, block_list: np.ndarray, block_count: np.ndarray,
                     scale: Optional[float] = None, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """``attention`` with q and k quantised to e4m3 per token (decided in fp32, as the
    FP8 attention kernel does) and v unchanged; the softmax weights stay exact."""
    qd, _ = quant_rows_e4m3_f32(q)
    kd, _ = quant_rows_e4m3_f32(k)
    vd = _bf16_bits(v).view(np.uint16).astype(np.uint32) << 16
    vd = vd.view(np.float32).astype(np.float64)
    return attention_f64(s, qd, kd, vd, block_list, block_count, scale=scale, rows=rows)


def quant_cols_e4m3(x, rows: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Per-channel e4m3 quantisation of bf16 x [B,H,stride,D] over the first `rows`
    rows of each head: (dequantised fp64 [B,H,stride,D], scales [B,H,D])."""
    xb = _bf16_bits(x)
    B, H, stride, D = xb.shape
    rows = stride if rows is None else rows
    out = np.zeros(xb.shape, np.float64)
    sc = np.zeros((B, H, D), np.float64)
    _load().orc_quant_cols_e4m3(_ptr(xb), B * H, rows, stride, D, _ptr(out), _ptr(sc))
    return out, sc


def attention_f64(s: Shape, q: np.ndarray, k: np.ndarray, v: np.ndarray, block_list: np.ndarray,
                  block_count: np.ndarray, scale: Optional[float] = None,
                  rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """``attention`` for fp64 inputs (q [B,H,Lq,D], k and v [B,H,kv_stride,D])."""
    lib = _load()
    qa, ka, va = (np.ascontiguousarray(a, np.float64) for a in (q, k, v))
    lst = np.ascontiguousarray(block_list, np.int32)
    cnt = np.ascontiguousarray(block_count, np.int32)
    cap = lst.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(s.head_dim)
    full = rows is None
    if full:
        rows = np.arange(s.batch * s.heads * s.Lq, dtype=np.int64)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((r.size, s.head_dim), np.float64)
    lib.orc_attention_f64(s.batch, s.heads, s.head_dim, s.frame_tokens, s.block_tokens, s.n_cur,
                          s.stride, _ptr(qa), _ptr(ka), _ptr(va), _ptr(lst), _ptr(cnt), cap,
                          float(scale), _ptr(r), r.size, _ptr(out))
    if full:
        return out.reshape(s.batch, s.heads, s.Lq, s.head_dim)
    return out


def attention_fp8_inputs(s: Shape, q, k, v, block_list: np.ndarray, block_count: np.ndarray,
                         scale: Optional[float] = None, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """``attention`` over e4m3-quantised inputs: q and k per token, v per channel of each
    head (over the call's n_frames * frame_tokens rows); the softmax weights stay exact."""
    qd, _ = quant_rows_e4m3(q)
    kd, _ = quant_rows_e4m3(k)
    vd, _ = quant_cols_e4m3(v, s.n_frames * s.frame_tokens)
    return attention_f64(s, qd, kd, vd, block_list, block_count, scale=scale, rows=rows)


def cag(T: Sequence[float], w: Optional[Sequence[float]], s_base: float, s_target: float,
        target_over_all: bool = True) -> Tuple[int, np.ndarray, float]:
    """Chunk-Aware Growth: (status, s[n], beta); status 0 = feasible."""
    lib = _load()
    Ta = np.ascontiguousarray(np.asarray(T, np.float64))
    n = Ta.size
    wa = np.ascontiguousarray(np.asarray(w if w is not None else np.arange(1, n + 1), np.float64))
    s_out = np.zeros(n, np.float64)
    beta = ctypes.c_double(0.0)
    rc = lib.orc_cag(n, _ptr(Ta), _ptr(wa), float(s_base), float(s_target),
                     1 if target_over_all else 0, _ptr(s_out), ctypes.byref(beta))
    return rc, s_out, beta.value


def blocks_for_sparsity(s: float, n_kv_blocks: int, n_sel: int, bpf: int) -> int:
    return _load().orc_blocks_for_sparsity(float(s), n_kv_blocks, n_sel, bpf)


def run_hsa(s: Shape, q, k, v, chunk_index: int, topk_frames: int, topk_blocks: int,
            scale: Optional[float] = None, rows: Optional[Sequence[int]] = None) -> dict:
    """The whole call in the pages' order: pool, select frames, select blocks, attend."""
    q_pool, k_pool, k_frame = pool(s, q, k)
    sel, fscores = select_frames(s, chunk_index, topk_frames, q_pool, k_frame)
    lst, cnt, bscores = select_blocks(s, chunk_index, topk_blocks, q_pool, k_pool, sel)
    out = attention(s, q, k, v, lst, cnt, scale, rows)
    return dict(q_pool=q_pool, k_pool=k_pool, k_frame=k_frame, frame_sel=sel,
                frame_scores=fscores, block_list=lst, block_count=cnt, block_scores=bscores,
                out=out)
