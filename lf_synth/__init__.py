"""Seeded synthetic inputs for the Light Forcing HSA call.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests and
benchmark. It only draws random tensors with the shapes and planted structure of
480p chunked video workloads; it performs none of the method's arithmetic (no
pooling, no scoring, no top-k, no budget solving). Every tensor is drawn in fp32
from a seeded ``torch.Generator`` on the CPU and rounded once to bf16, so both
sides receive the same bf16 bytes.

Shapes follow the pages' 480p setting: a 30x52 latent grid gives 1560 tokens per
frame, chunks are 3 frames, 12 heads of dimension 128 ("Light Forcing:
Accelerating Autoregressive Video Diffusion via Sparse Attention", gist.science,
Technical Summary section 2.2, and the chunk experiments of the 163.com article,
section 1). The planted structures stand in for the attention patterns the pages
describe (diagonal / same-position locality, attention sinks, a relevant distant
memory frame; 163.com article section 3, attention-visualisation paragraph).
The VBench prompts and trained weights the pages evaluate with are not available;
these inputs stand in for them.

Layout of every tensor: [batch, heads, tokens, head_dim], contiguous, bf16. KV
frames are ordered [sink..., memory..., recent..., current chunk...] in time
order; queries are the current-chunk frames.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import torch

__all__ = ["Workload", "CONFIGS", "make_qkv", "make_rollout_qkv", "workload"]


@dataclass(frozen=True)
class Workload:
    """One HSA call's sizes and hyper-parameters (no derived quantities).

    ``sparsity`` is the target block sparsity the caller wants; turning it into
    a per-frame block count is method arithmetic and lives on each side, not here.
    ``topk_blocks`` overrides it when a config fixes the count directly.
    """

    name: str
    batch: int
    heads: int
    head_dim: int
    frame_tokens: int
    block_tokens: int
    n_sink: int
    n_mem: int
    n_recent: int
    n_cur: int
    topk_frames: int
    sparsity: Optional[float] = None
    topk_blocks: Optional[int] = None
    chunk_index: int = 2
    seed: int = 0
    recipe: str = "noise"
    extra: Dict[str, float] = field(default_factory=dict)

    @property
    def n_frames(self) -> int:
        return self.n_sink + self.n_mem + self.n_recent + self.n_cur

    @property
    def q_tokens(self) -> int:
        return self.n_cur * self.frame_tokens

    @property
    def kv_tokens(self) -> int:
        return self.n_frames * self.frame_tokens


# The five workloads: tiny parity case, one 480p layer call, the chunk rollout
# (per-chunk shapes come from ``make_rollout_qkv``), long-video retrieval stress,
# and a two-sequence batch with per-head planted patterns.
CONFIGS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 64, 256, 64, 1, 5, 1, 2, topk_frames=2,
                     topk_blocks=2, seed=0, recipe="planted_means"),
    "layer480p": Workload("layer480p", 1, 12, 128, 1560, 64, 1, 16, 1, 3,
                          topk_frames=4, sparsity=0.80, seed=1,
                          recipe="planted_means_diagonal"),
    "rollout480p": Workload("rollout480p", 1, 12, 128, 1560, 64, 1, 16, 1, 3,
                            topk_frames=4, sparsity=0.80, seed=2,
                            recipe="rollout", extra={"n_chunks": 7, "s_base": 0.95}),
    "longvideo480p": Workload("longvideo480p", 1, 12, 128, 1560, 64, 1, 60, 1, 3,
                              topk_frames=4, sparsity=0.90, seed=3, recipe="low_rank"),
    "patterns480p": Workload("patterns480p", 2, 12, 128, 1560, 64, 1, 16, 1, 3,
                             topk_frames=4, sparsity=0.80, seed=4,
                             recipe="head_patterns"),
}


def workload(name: str, **overrides) -> Workload:
    """Return a named workload, optionally with fields replaced."""
    return replace(CONFIGS[name], **overrides)


def _unit_rows(g: torch.Generator, n: int, d: int) -> torch.Tensor:
    x = torch.randn(n, d, generator=g, dtype=torch.float32)
    return x / x.norm(dim=1, keepdim=True)


def _to_bf16(*ts: torch.Tensor) -> Tuple[torch.Tensor, ...]:
    return tuple(t.to(torch.bfloat16).contiguous() for t in ts)


def _frame_view(x: torch.Tensor, frame_tokens: int) -> torch.Tensor:
    b, h, l, d = x.shape
    return x.view(b, h, l // frame_tokens, frame_tokens, d)


def _add_to_query_blocks(q: torch.Tensor, w: Workload, vec_for) -> None:
    """Add vec_for(b, h, r) (a [D] tensor or None) to every token of query block r.

    Query block r is the j-th 64-token block of current-chunk frame f, with
    r = f * ceil(F/64) + j; blocks never cross frame boundaries.
    """
    bt, F = w.block_tokens, w.frame_tokens
    bpf = -(-F // bt)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            for f in range(q.shape[2] // F):
                for j in range(bpf):
                    r = f * bpf + j
                    vec = vec_for(b, h, r)
                    if vec is None:
                        continue
                    t0 = f * F + j * bt
                    t1 = f * F + min((j + 1) * bt, F)
                    q[b, h, t0:t1, :] += vec


def _diagonal_bias(g: torch.Generator, heads: int, F: int, D: int) -> torch.Tensor:
    # One vector per (head, spatial position) with squared norm sqrt(D), so a
    # query and a key at the same position gain about +1 logit after 1/sqrt(D).
    return _unit_rows(g, heads * F, D).view(heads, F, D) * (D ** 0.25)


def make_qkv(w: Workload, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Draw (q, k, v) for one HSA call of workload ``w``.

    Draw order (fixed, so the bytes are reproducible): q, k, v ~ N(0, 1) in that
    order, then the recipe's planted vectors.
    """
    g = torch.Generator().manual_seed(w.seed)
    B, H, D, F = w.batch, w.heads, w.head_dim, w.frame_tokens
    q = torch.randn(B, H, w.q_tokens, D, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, w.kv_tokens, D, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, w.kv_tokens, D, generator=g, dtype=torch.float32)
    kf = _frame_view(k, F)
    mem0 = w.n_sink

    if w.recipe in ("planted_means", "planted_means_diagonal"):
        # Per-frame mean vector of norm 2 on every memory frame's keys; the even
        # query blocks carry the mean of one memory frame ("half the query blocks
        # align").
        u = _unit_rows(g, B * H * max(w.n_mem, 1), D).view(B, H, max(w.n_mem, 1), D) * 2.0
        for m in range(w.n_mem):
            kf[:, :, mem0 + m, :, :] += u[:, :, m, None, :]
        if w.n_mem > 0:
            def vec_for(b, h, r):
                if r % 2:
                    return None
                if w.recipe == "planted_means":
                    m = (r // 2) % w.n_mem
                else:
                    m = (r * 7 + h) % w.n_mem
                return u[b, h, m]
            _add_to_query_blocks(q, w, vec_for)
        if w.recipe == "planted_means_diagonal":
            c = _diagonal_bias(g, H, F, D)
            _frame_view(q, F)[:] += c[None, :, None, :, :]
            kf[:] += c[None, :, None, :, :]
    elif w.recipe == "low_rank":
        # Rank-8 structure: keys of frame f get a_{h,f} W_h, query block r gets
        # c_{h,r} W_h, with W_h having orthonormal rows.
        rank = 8
        W = torch.linalg.qr(torch.randn(H, D, rank, generator=g, dtype=torch.float32))[0]
        W = W.transpose(1, 2).contiguous()  # [H, rank, D], orthonormal rows
        a = torch.randn(B, H, w.n_frames, rank, generator=g, dtype=torch.float32) * (2.0 / math.sqrt(rank))
        kf[:] += torch.einsum("bhfr,hrd->bhfd", a, W)[:, :, :, None, :]
        bpf = -(-F // w.block_tokens)
        cq = torch.randn(B, H, w.n_cur * bpf, rank, generator=g, dtype=torch.float32) * (2.0 / math.sqrt(rank))
        cW = torch.einsum("bhrk,hkd->bhrd", cq, W)
        _add_to_query_blocks(q, w, lambda b, h, r: cW[b, h, r])
    elif w.recipe == "head_patterns":
        # Head h gets pattern h mod 4: (0) sink on frame 0, (1) diagonal spatial
        # locality, (2) one distant memory frame (the oldest), (3) plain noise.
        # Keys are then scaled x4 to sharpen the softmax.
        gvec = _unit_rows(g, B * H, D).view(B, H, D) * 2.0
        c = _diagonal_bias(g, H, F, D)
        for h in range(H):
            p = h % 4
            if p == 0:
                kf[:, h, 0, :, :] += gvec[:, h, None, :]
                q[:, h] += gvec[:, h, None, :]
            elif p == 1:
                _frame_view(q, F)[:, h] += c[h][None, None, :, :]
                kf[:, h] += c[h][None, None, :, :]
            elif p == 2 and w.n_mem > 0:
                kf[:, h, mem0, :, :] += gvec[:, h, None, :]
                q[:, h] += gvec[:, h, None, :]
        k *= 4.0
    elif w.recipe == "noise":
        pass
    else:
        raise ValueError(f"unknown recipe {w.recipe!r}")

    q, k, v = _to_bf16(q, k, v)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def make_rollout_qkv(w: Workload) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Draw the whole rollout once: q, k, v for all n_chunks * n_cur frames.

    Chunk i (1-based) attends with queries = frames [n_cur*(i-1), n_cur*i) and
    KV = frames [0, n_cur*i). Keys of every frame f >= 1 carry a planted mean of
    norm 2; even query blocks of chunk i >= 2 carry the mean of one earlier
    non-sink frame; a diagonal bias is added to q and k as in ``layer480p``.
    """
    g = torch.Generator().manual_seed(w.seed)
    n_chunks = int(w.extra.get("n_chunks", 7))
    B, H, D, F, C = w.batch, w.heads, w.head_dim, w.frame_tokens, w.n_cur
    n_fr = n_chunks * C
    L = n_fr * F
    q = torch.randn(B, H, L, D, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, L, D, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, L, D, generator=g, dtype=torch.float32)
    u = _unit_rows(g, B * H * n_fr, D).view(B, H, n_fr, D) * 2.0
    kf = _frame_view(k, F)
    kf[:, :, 1:, :, :] += u[:, :, 1:, None, :]
    bpf = -(-F // w.block_tokens)
    qf = _frame_view(q, F)
    for b in range(B):
        for h in range(H):
            for fq in range(C, n_fr):
                chunk = fq // C + 1
                n_hist = C * (chunk - 1)      # frames before this chunk
                span = max(1, n_hist - 1)      # non-sink history frames
                for j in range(0, bpf):
                    r = (fq % C) * bpf + j
                    if r % 2:
                        continue
                    m = 1 + (r * 7 + h) % span
                    t0, t1 = j * w.block_tokens, min((j + 1) * w.block_tokens, F)
                    qf[b, h, fq, t0:t1, :] += u[b, h, m]
    c = _diagonal_bias(g, H, F, D)
    qf[:] += c[None, :, None, :, :]
    kf[:] += c[None, :, None, :, :]
    return _to_bf16(q, k, v)


def rollout_chunk(w: Workload, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, chunk: int):
    """Slice chunk ``chunk`` (1-based) out of a rollout drawn by make_rollout_qkv.

    Returns (workload, q, k, v) with contiguous tensors and the frame roles of
    that chunk: chunk 1 has only its own frames; chunk i >= 2 has 1 sink frame,
    n_cur*(i-1)-2 memory frames, 1 recent frame and the current chunk.
    """
    C, F = w.n_cur, w.frame_tokens
    n_kv_fr = C * chunk
    if chunk == 1:
        roles = dict(n_sink=0, n_mem=0, n_recent=0, n_cur=C)
    else:
        roles = dict(n_sink=1, n_mem=n_kv_fr - C - 2, n_recent=1, n_cur=C)
    wc = replace(w, chunk_index=chunk, **roles)
    qs = q[:, :, (chunk - 1) * C * F: chunk * C * F, :].contiguous()
    ks = k[:, :, : n_kv_fr * F, :].contiguous()
    vs = v[:, :, : n_kv_fr * F, :].contiguous()
    return wc, qs, ks, vs
