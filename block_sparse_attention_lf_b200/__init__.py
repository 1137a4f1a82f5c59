"""Python binding of liblf_hsa.so, the B200 Light Forcing HSA library.

Argument marshalling only: every step of the HSA call runs in the library's
CUDA kernels (sm_100a). PyTorch supplies device memory and the current stream.
The functions carry the C names (``lf_pool``, ``lf_select_frames``,
``lf_select_blocks``, ``lf_block_sparse_attn``, ``lf_cag_budget``, ...) and
take preallocated torch tensors; ``HSACall`` is a convenience wrapper that
allocates the intermediate buffers and runs the four device steps in order.

The library is loaded from this directory (``liblf_hsa.so``, built by
``build.py``); importing this module fails loudly when it is missing, and the
device entry points raise when the tensors are not CUDA tensors. There is no
CPU fallback.

Typical use (q [B,H,n_cur*F,D], k and v [B,H,n_frames*F,D], bf16 on the GPU)::

    shape = LfShape.make(B, H, D, F, n_frames, n_sink, n_recent, n_cur)
    call = HSACall(shape, chunk_index, topk_frames, topk_blocks)
    out = call(q, k, v)          # pool, select frames, select blocks, attend

``HSACall.attend`` uses ``lf_block_sparse_attn_ws`` with a workspace sized by
``lf_attn_split_plan`` (the split of the attention's last, partial wave);
``tail_pieces=1`` turns the split off. ``lf_pool_range`` re-pools only some
frames (keep the pooled keys of past frames between calls),
``lf_select_blocks_1d`` gives the single-granularity lists of the ablation, and
``lf_cag_budget`` / ``lf_blocks_for_sparsity`` turn a sparsity target into
per-chunk block counts.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblf_hsa.so")

__all__ = [
    "LfShape", "LfError", "lib", "lf_pool", "lf_pool_range", "lf_select_frames", "lf_select_blocks",
    "lf_select_blocks_1d", "lf_frame_index_build", "lf_select_frames_ivf", "FrameIndex", "lf_select_mask",
    "lf_quant_fp8_rows", "lf_block_sparse_attn_fp8",
    "lf_block_sparse_attn", "lf_block_sparse_attn_ws", "lf_attn_split_plan", "lf_cag_budget",
    "lf_blocks_for_sparsity", "lf_frames_selected", "lf_list_capacity", "lf_get_device_error",
    "lf_status_string", "lf_version", "HSACall",
    "ABI_FUNCTIONS", "shard_units", "shard_shape", "unit_view",
]

# Names declared in include/lf_hsa.h.
ABI_FUNCTIONS = (
    "lf_pool", "lf_pool_range", "lf_frames_selected", "lf_select_frames", "lf_list_capacity", "lf_select_blocks",
    "lf_select_blocks_1d", "lf_frame_index_build", "lf_select_frames_ivf", "lf_select_mask", "lf_quant_fp8_rows",
    "lf_block_sparse_attn_fp8",
    "lf_block_sparse_attn", "lf_block_sparse_attn_ws", "lf_attn_split_plan", "lf_block_sparse_attn_static",
    "lf_cag_budget", "lf_blocks_for_sparsity", "lf_get_device_error", "lf_status_string", "lf_version",
)

LF_OK = 0
STATUS_NAMES = {
    0: "LF_OK", 1: "LF_ERR_NULL", 2: "LF_ERR_ALIGN", 3: "LF_ERR_SHAPE", 4: "LF_ERR_TOPK",
    5: "LF_ERR_CAP", 6: "LF_ERR_INFEASIBLE", 7: "LF_ERR_CUDA", 8: "LF_ERR_DEVICE_TIMEOUT",
    9: "LF_ERR_ARG", 10: "LF_ERR_LIST", 11: "LF_ERR_NO_DEVICE", 12: "LF_ERR_SCRATCH",
}


class LfError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_lib.lf_status_string(status).decode()})")


class LfShape(ctypes.Structure):
    """Mirror of ``lf_hsa_shape``."""

    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("frame_tokens", ctypes.c_int32), ("block_tokens", ctypes.c_int32),
        ("n_frames", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("n_recent", ctypes.c_int32),
        ("n_cur", ctypes.c_int32), ("kv_stride", ctypes.c_int64),
    ]

    @classmethod
    def make(cls, batch, heads, head_dim, frame_tokens, n_frames, n_sink, n_recent, n_cur,
             block_tokens=64, kv_stride=0) -> "LfShape":
        return cls(batch, heads, head_dim, frame_tokens, block_tokens, n_frames, n_sink, n_recent,
                   n_cur, kv_stride)

    @property
    def bpf(self) -> int:
        return -(-self.frame_tokens // self.block_tokens)

    @property
    def Rq(self) -> int:
        return self.n_cur * self.bpf

    @property
    def Nkv(self) -> int:
        return self.n_frames * self.bpf

    @property
    def Lq(self) -> int:
        return self.n_cur * self.frame_tokens

    @property
    def Lkv(self) -> int:
        return self.n_frames * self.frame_tokens


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_lf_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, F32, F64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_double
    S = ctypes.POINTER(LfShape)
    sig = {
        "lf_pool": ([S, P, P, P, P, P, P], I32),
        "lf_pool_range": ([S, P, P, I32, I32, I32, P, P, P, P], I32),
        "lf_frames_selected": ([S, I32, I32], I32),
        "lf_select_frames": ([S, I32, I32, P, P, P, P], I32),
        "lf_list_capacity": ([S, I32, I32, I32], I32),
        "lf_select_blocks": ([S, I32, I32, I32, P, P, P, P, P, I32, P], I32),
        "lf_select_blocks_1d": ([S, I32, I32, P, P, P, P, I32, P], I32),
        "lf_frame_index_build": ([S, I32, I32, P, P, P, P, P, P], I32),
        "lf_select_mask": ([S, I32, I32, I32, P, P, P, P, P, P, I32, P], I32),
        "lf_quant_fp8_rows": ([P, ctypes.c_int64, I32, P, P, P], I32),
        "lf_block_sparse_attn_fp8": ([S, P, P, P, P, P, P, P, I32, F32, P, I32, P, ctypes.c_int64, P], I32),
        "lf_select_frames_ivf": ([S, I32, I32, I32, I32, P, P, P, P, P, P, P], I32),
        "lf_block_sparse_attn": ([S, P, P, P, P, P, I32, F32, P, P], I32),
        "lf_block_sparse_attn_ws": ([S, P, P, P, P, P, I32, F32, P, I32, P, ctypes.c_int64, P], I32),
        "lf_attn_split_plan": ([S, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32),
                                ctypes.POINTER(ctypes.c_int64)], I32),
        "lf_block_sparse_attn_static": ([S, P, P, P, P, P, I32, F32, P, I32, P], I32),
        "lf_cag_budget": ([I32, P, P, F64, F64, I32, P, P], I32),
        "lf_blocks_for_sparsity": ([F64, I32, I32, I32], I32),
        "lf_get_device_error": ([ctypes.POINTER(I32)], I32),
        "lf_status_string": ([I32], ctypes.c_char_p),
        "lf_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


_lib = _load()
lib = _lib


def _check(status: int, where: str) -> None:
    if status != LF_OK:
        raise LfError(status, where)


def _dev_ptr(t, dtype, name: str):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _bf16():
    import torch
    return torch.bfloat16


def lf_version() -> str:
    return _lib.lf_version().decode()


def lf_status_string(status: int) -> str:
    return _lib.lf_status_string(status).decode()


def lf_frames_selected(shape: LfShape, chunk_index: int, topk_frames: int) -> int:
    return _lib.lf_frames_selected(ctypes.byref(shape), chunk_index, topk_frames)


def lf_list_capacity(shape: LfShape, chunk_index: int, topk_frames: int, topk_blocks: int) -> int:
    return _lib.lf_list_capacity(ctypes.byref(shape), chunk_index, topk_frames, topk_blocks)


def lf_blocks_for_sparsity(s: float, n_kv_blocks: int, n_sel_frames: int, bpf: int) -> int:
    return _lib.lf_blocks_for_sparsity(float(s), n_kv_blocks, n_sel_frames, bpf)


def lf_pool_range(shape: LfShape, q, k, frame_begin: int, frame_end: int, q_pool, k_pool, k_frame,
                  pool_q: bool = True, stream=None) -> None:
    """Pool KV frames [frame_begin, frame_end) (and q when ``pool_q``) into the
    same buffers lf_pool fills; other entries are left as they are."""
    import torch
    bf = _bf16()
    qp = _dev_ptr(q, bf, "q") if pool_q else None
    qpp = _dev_ptr(q_pool, torch.float32, "q_pool") if pool_q else None
    _check(_lib.lf_pool_range(ctypes.byref(shape), qp, _dev_ptr(k, bf, "k"), int(frame_begin), int(frame_end),
                              1 if pool_q else 0, qpp, _dev_ptr(k_pool, torch.float32, "k_pool"),
                              _dev_ptr(k_frame, torch.float32, "k_frame"), _stream(stream)), "lf_pool_range")


def lf_pool(shape: LfShape, q, k, q_pool, k_pool, k_frame, stream=None) -> None:
    import torch
    bf = _bf16()
    _check(_lib.lf_pool(ctypes.byref(shape), _dev_ptr(q, bf, "q"), _dev_ptr(k, bf, "k"),
                        _dev_ptr(q_pool, torch.float32, "q_pool"),
                        _dev_ptr(k_pool, torch.float32, "k_pool"),
                        _dev_ptr(k_frame, torch.float32, "k_frame"), _stream(stream)), "lf_pool")


def lf_select_frames(shape: LfShape, chunk_index: int, topk_frames: int, q_pool, k_frame,
                     frame_sel, stream=None) -> None:
    import torch
    _check(_lib.lf_select_frames(ctypes.byref(shape), chunk_index, topk_frames,
                                 _dev_ptr(q_pool, torch.float32, "q_pool"),
                                 _dev_ptr(k_frame, torch.float32, "k_frame"),
                                 _dev_ptr(frame_sel, torch.int32, "frame_sel"), _stream(stream)),
           "lf_select_frames")


def lf_select_blocks(shape: LfShape, chunk_index: int, topk_frames: int, topk_blocks: int, q_pool,
                     k_pool, frame_sel, block_list, block_count, list_cap: int, stream=None) -> None:
    import torch
    _check(_lib.lf_select_blocks(ctypes.byref(shape), chunk_index, topk_frames, topk_blocks,
                                 _dev_ptr(q_pool, torch.float32, "q_pool"),
                                 _dev_ptr(k_pool, torch.float32, "k_pool"),
                                 _dev_ptr(frame_sel, torch.int32, "frame_sel"),
                                 _dev_ptr(block_list, torch.int32, "block_list"),
                                 _dev_ptr(block_count, torch.int32, "block_count"), list_cap,
                                 _stream(stream)), "lf_select_blocks")


def lf_select_mask(shape: LfShape, chunk_index: int, topk_frames: int, topk_blocks: int, q_pool, k_frame, k_pool,
                   frame_sel, block_list, block_count, list_cap: int, stream=None) -> None:
    """Both selection levels in one launch (the results of lf_select_frames + lf_select_blocks)."""
    import torch
    f32, i32 = torch.float32, torch.int32
    _check(_lib.lf_select_mask(ctypes.byref(shape), chunk_index, topk_frames, topk_blocks,
                               _dev_ptr(q_pool, f32, "q_pool"), _dev_ptr(k_frame, f32, "k_frame"),
                               _dev_ptr(k_pool, f32, "k_pool"), _dev_ptr(frame_sel, i32, "frame_sel"),
                               _dev_ptr(block_list, i32, "block_list"), _dev_ptr(block_count, i32, "block_count"),
                               list_cap, _stream(stream)), "lf_select_mask")


def lf_quant_fp8_rows(x, x8, scales, stream=None) -> None:
    """Per-row e4m3 codes (uint8 tensor shaped like x) and fp32 scales (x.shape[:-1]) of bf16 x."""
    import torch
    D = x.shape[-1]
    n = x.numel() // D
    _check(_lib.lf_quant_fp8_rows(_dev_ptr(x, _bf16(), "x"), n, D, _dev_ptr(x8, torch.uint8, "x8"),
                                  _dev_ptr(scales, torch.float32, "scales"), _stream(stream)), "lf_quant_fp8_rows")


def lf_select_blocks_1d(shape: LfShape, chunk_index: int, topk_blocks: int, q_pool, k_pool,
                        block_list, block_count, list_cap: int, stream=None) -> None:
    import torch
    _check(_lib.lf_select_blocks_1d(ctypes.byref(shape), chunk_index, topk_blocks,
                                    _dev_ptr(q_pool, torch.float32, "q_pool"),
                                    _dev_ptr(k_pool, torch.float32, "k_pool"),
                                    _dev_ptr(block_list, torch.int32, "block_list"),
                                    _dev_ptr(block_count, torch.int32, "block_count"), list_cap,
                                    _stream(stream)), "lf_select_blocks_1d")


@dataclass
class FrameIndex:
    """Device buffers of a coarse frame index (lf_frame_index_build): fp32 centroids
    [B,H,n_clusters,D], int32 labels and members [B,H,max(n_mem,1)], int32 offsets
    [B,H,n_clusters+1]."""
    n_clusters: int
    centroids: "object"
    labels: "object"
    offsets: "object"
    members: "object"

    @classmethod
    def empty(cls, shape: LfShape, n_clusters: int, device="cuda") -> "FrameIndex":
        import torch
        n_mem = max(shape.n_frames - shape.n_sink - shape.n_recent - shape.n_cur, 1)
        bh = (shape.batch, shape.heads)
        return cls(n_clusters,
                   torch.empty(*bh, n_clusters, shape.head_dim, dtype=torch.float32, device=device),
                   torch.empty(*bh, n_mem, dtype=torch.int32, device=device),
                   torch.empty(*bh, n_clusters + 1, dtype=torch.int32, device=device),
                   torch.empty(*bh, n_mem, dtype=torch.int32, device=device))


def lf_frame_index_build(shape: LfShape, k_frame, index: FrameIndex, iters: int = 25, stream=None) -> None:
    """k-means index over each head's memory-frame means (k_frame from lf_pool)."""
    import torch
    i32 = torch.int32
    _check(_lib.lf_frame_index_build(ctypes.byref(shape), int(index.n_clusters), int(iters),
                                     _dev_ptr(k_frame, torch.float32, "k_frame"),
                                     _dev_ptr(index.centroids, torch.float32, "centroids"),
                                     _dev_ptr(index.labels, i32, "labels"), _dev_ptr(index.offsets, i32, "offsets"),
                                     _dev_ptr(index.members, i32, "members"), _stream(stream)),
           "lf_frame_index_build")


def lf_select_frames_ivf(shape: LfShape, chunk_index: int, topk_frames: int, index: FrameIndex, n_probe: int,
                         q_pool, k_frame, frame_sel, stream=None) -> None:
    """Frame selection probing the index (same output layout as lf_select_frames)."""
    import torch
    i32 = torch.int32
    _check(_lib.lf_select_frames_ivf(ctypes.byref(shape), chunk_index, topk_frames, int(index.n_clusters),
                                     int(n_probe), _dev_ptr(q_pool, torch.float32, "q_pool"),
                                     _dev_ptr(k_frame, torch.float32, "k_frame"),
                                     _dev_ptr(index.centroids, torch.float32, "centroids"),
                                     _dev_ptr(index.offsets, i32, "offsets"), _dev_ptr(index.members, i32, "members"),
                                     _dev_ptr(frame_sel, i32, "frame_sel"), _stream(stream)),
           "lf_select_frames_ivf")


def lf_block_sparse_attn(shape: LfShape, q, k, v, block_list, block_count, list_cap: int,
                         softmax_scale: float, out, stream=None) -> None:
    import torch
    bf = _bf16()
    _check(_lib.lf_block_sparse_attn(ctypes.byref(shape), _dev_ptr(q, bf, "q"), _dev_ptr(k, bf, "k"),
                                     _dev_ptr(v, bf, "v"),
                                     _dev_ptr(block_list, torch.int32, "block_list"),
                                     _dev_ptr(block_count, torch.int32, "block_count"), list_cap,
                                     float(softmax_scale), _dev_ptr(out, bf, "out"), _stream(stream)),
           "lf_block_sparse_attn")


def lf_block_sparse_attn_ws(shape: LfShape, q, k, v, block_list, block_count, list_cap: int,
                            softmax_scale: float, out, workspace=None, tail_pieces: int = 0,
                            stream=None) -> None:
    """``workspace``: a uint8 device tensor (or None: no split)."""
    import torch
    bf = _bf16()
    ws = _dev_ptr(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(_lib.lf_block_sparse_attn_ws(ctypes.byref(shape), _dev_ptr(q, bf, "q"), _dev_ptr(k, bf, "k"),
                                        _dev_ptr(v, bf, "v"),
                                        _dev_ptr(block_list, torch.int32, "block_list"),
                                        _dev_ptr(block_count, torch.int32, "block_count"), list_cap,
                                        float(softmax_scale), _dev_ptr(out, bf, "out"), int(tail_pieces),
                                        ws, ws_bytes, _stream(stream)),
           "lf_block_sparse_attn_ws")


def lf_block_sparse_attn_fp8(shape: LfShape, q8, k8, q_scale, k_scale, v, block_list, block_count, list_cap: int,
                             softmax_scale: float, out, workspace=None, tail_pieces: int = 0, stream=None) -> None:
    """Attention with e4m3 q8 / k8 (uint8 codes from lf_quant_fp8_rows) and fp32 per-token scales."""
    import torch
    bf = _bf16()
    u8, f32, i32 = torch.uint8, torch.float32, torch.int32
    ws = _dev_ptr(workspace, u8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(_lib.lf_block_sparse_attn_fp8(ctypes.byref(shape), _dev_ptr(q8, u8, "q8"), _dev_ptr(k8, u8, "k8"),
                                         _dev_ptr(q_scale, f32, "q_scale"), _dev_ptr(k_scale, f32, "k_scale"),
                                         _dev_ptr(v, bf, "v"), _dev_ptr(block_list, i32, "block_list"),
                                         _dev_ptr(block_count, i32, "block_count"), list_cap, float(softmax_scale),
                                         _dev_ptr(out, bf, "out"), int(tail_pieces), ws, ws_bytes, _stream(stream)),
           "lf_block_sparse_attn_fp8")


def lf_attn_split_plan(shape: LfShape, list_cap: int, sm: int = 0) -> Tuple[int, int, int]:
    """(tail query blocks, pieces per list, workspace bytes) of the automatic split."""
    t, p, b = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int64(0)
    _check(_lib.lf_attn_split_plan(ctypes.byref(shape), list_cap, sm, ctypes.byref(t), ctypes.byref(p),
                                   ctypes.byref(b)), "lf_attn_split_plan")
    return t.value, p.value, b.value


def lf_cag_budget(T: Sequence[float], flops_w: Optional[Sequence[float]], s_base: float,
                  s_target: float, target_over_all: bool = True) -> Tuple[int, list, float]:
    """Host-only Chunk-Aware Growth solver: returns (status, s[n], beta)."""
    n = len(T)
    Ta = (ctypes.c_double * n)(*[float(x) for x in T])
    wa = (ctypes.c_double * n)(*[float(x) for x in flops_w]) if flops_w is not None else None
    s_out = (ctypes.c_double * max(n, 1))()
    beta = ctypes.c_double(0.0)
    st = _lib.lf_cag_budget(n, ctypes.cast(Ta, ctypes.c_void_p),
                            ctypes.cast(wa, ctypes.c_void_p) if wa is not None else None,
                            float(s_base), float(s_target), 1 if target_over_all else 0,
                            ctypes.cast(s_out, ctypes.c_void_p), ctypes.byref(beta))
    return st, list(s_out)[:n], beta.value


def lf_get_device_error() -> Tuple[int, int]:
    """(status, detail) of the current device's error word; clears it."""
    d = ctypes.c_int32(0)
    st = _lib.lf_get_device_error(ctypes.byref(d))
    return st, d.value


@dataclass
class HSABuffers:
    q_pool: "object"
    k_pool: "object"
    k_frame: "object"
    frame_sel: "object"
    block_list: "object"
    block_count: "object"
    out: "object"
    list_cap: int


class HSACall:
    """One HSA call's device buffers plus the device steps, in order: pooling, the
    two-level selection (one launch, lf_select_mask) and the attention.

    ``shape``: an ``LfShape``; ``chunk_index`` is 1-based (chunk 1 is dense);
    ``topk_frames`` / ``topk_blocks`` as in the C ABI. ``tail_pieces`` selects
    the attention's split of the last, partial wave (0: automatic plan for the
    current device, 1: none, k >= 2: k pieces); the workspace it needs is
    allocated here.
    """

    def __init__(self, shape: LfShape, chunk_index: int, topk_frames: int, topk_blocks: int,
                 device="cuda", softmax_scale: float = 0.0, tail_pieces: int = 0):
        import torch
        self.shape, self.chunk_index = shape, chunk_index
        self.topk_frames, self.topk_blocks = topk_frames, topk_blocks
        self.softmax_scale = softmax_scale
        s = shape
        D = s.head_dim
        n_sel = lf_frames_selected(s, chunk_index, topk_frames)
        cap = lf_list_capacity(s, chunk_index, topk_frames, topk_blocks)
        if n_sel < 0 or cap < 0:
            raise LfError(3, "HSACall")
        self.n_sel = n_sel
        f32, i32 = torch.float32, torch.int32
        self.buf = HSABuffers(
            q_pool=torch.empty(s.batch, s.heads, s.Rq, D, dtype=f32, device=device),
            k_pool=torch.empty(s.batch, s.heads, s.Nkv, D, dtype=f32, device=device),
            k_frame=torch.empty(s.batch, s.heads, s.n_frames, D, dtype=f32, device=device),
            frame_sel=torch.empty(s.batch, s.heads, s.Rq, n_sel, dtype=i32, device=device),
            block_list=torch.empty(s.batch, s.heads, s.Rq, cap, dtype=i32, device=device),
            block_count=torch.empty(s.batch, s.heads, s.Rq, dtype=i32, device=device),
            out=torch.empty(s.batch, s.heads, s.Lq, D, dtype=torch.bfloat16, device=device),
            list_cap=cap,
        )
        self.tail_pieces = tail_pieces
        if tail_pieces == 0:
            tail, pieces, _ = lf_attn_split_plan(s, cap)
        elif tail_pieces >= 2:
            # the same tail as the automatic plan, with the piece count given
            sm = torch.cuda.get_device_properties(torch.device(device)).multi_processor_count
            tail = (s.batch * s.heads * s.Rq) % sm
            pieces = min(tail_pieces, cap)
            if pieces < 2:
                tail, pieces = 0, 0
        else:
            tail, pieces = 0, 0
        ws_bytes = tail * pieces * 64 * (D + 2) * 4
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes else None
        self.split = (tail, pieces) if ws_bytes else (0, 0)
        # kernels enqueued per call: pool, selection (both levels), attention (+ the merge of a split)
        self.launches_per_call = 3 + (1 if ws_bytes else 0)

    def pool(self, q, k, stream=None):
        b = self.buf
        lf_pool(self.shape, q, k, b.q_pool, b.k_pool, b.k_frame, stream)

    def select(self, stream=None):
        b = self.buf
        lf_select_mask(self.shape, self.chunk_index, self.topk_frames, self.topk_blocks, b.q_pool, b.k_frame,
                       b.k_pool, b.frame_sel, b.block_list, b.block_count, b.list_cap, stream)

    def attend(self, q, k, v, stream=None):
        b = self.buf
        lf_block_sparse_attn_ws(self.shape, q, k, v, b.block_list, b.block_count, b.list_cap,
                                self.softmax_scale, b.out, self.workspace, self.tail_pieces, stream)

    def __call__(self, q, k, v, stream=None):
        self.pool(q, k, stream)
        self.select(stream)
        self.attend(q, k, v, stream)
        return self.buf.out


def shard_units(batch: int, heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous range [u0, u1) of the call's batch*heads (batch, head) units that
    process ``rank`` of ``world`` takes. Pooling, selection and attention of one unit
    never read another unit's data, so the ranges need no exchange; their sizes
    differ by at most one unit, and a rank past the unit count gets an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    n = batch * heads
    return rank * n // world, (rank + 1) * n // world


def shard_shape(shape: LfShape, world: int, rank: int) -> Tuple[Optional[LfShape], int, int]:
    """(per-rank shape, u0, u1): the units [u0, u1) of ``shape`` as a call of their
    own (batch 1, u1 - u0 heads, same frames and head stride); None when the range
    is empty. The [B, H, L, D] tensors are contiguous over (batch, head), so the
    slice is a pointer offset (``unit_view``)."""
    u0, u1 = shard_units(shape.batch, shape.heads, world, rank)
    if u1 == u0:
        return None, u0, u1
    s = LfShape.make(1, u1 - u0, shape.head_dim, shape.frame_tokens, shape.n_frames, shape.n_sink,
                     shape.n_recent, shape.n_cur, block_tokens=shape.block_tokens, kv_stride=shape.kv_stride)
    return s, u0, u1


def unit_view(t, u0: int, u1: int):
    """Units [u0, u1) of a contiguous [B, H, L, D] tensor as a [1, u1 - u0, L, D] view."""
    if not t.is_contiguous():
        raise ValueError("unit_view needs a contiguous tensor")
    return t.reshape(-1, t.shape[-2], t.shape[-1])[u0:u1].unsqueeze(0)


def shape_from_workload(w) -> LfShape:
    """LfShape of an ``lf_synth.Workload`` (or anything with the same fields)."""
    return LfShape.make(w.batch, w.heads, w.head_dim, w.frame_tokens, w.n_frames, w.n_sink,
                        w.n_recent, w.n_cur, block_tokens=w.block_tokens)
