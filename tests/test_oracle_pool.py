"""Pins for the oracle's token compression (block and frame mean pooling).

Source: Light Forcing (paper.rainbus.top), execution flow, stage 2; gist.science
Technical Summary 2.2 "Token Compression". Each test checks the oracle against
something other than itself: a hand-worked example, a closed form, or an
identity between independently computed quantities.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    t = torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(a, np.float32))), "fixture not bf16-exact"
    return t


def test_pool_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "pool_hand.json")))
    s = oracle.Shape(**g["shape"])
    q = _bf16(g["q"]).reshape(1, 1, -1, 2)
    k = _bf16(g["k"]).reshape(1, 1, -1, 2)
    qp, kp, kf = oracle.pool(s, q, k)
    np.testing.assert_allclose(qp.reshape(-1, 2), g["q_pool"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(kp.reshape(-1, 2), g["k_pool"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(kf.reshape(-1, 2), g["k_frame"], rtol=0, atol=1e-15)


def test_pool_ramp_closed_form():
    """Token value = its index within the head plus a per-head/per-dim offset.

    Block mean = midpoint of the block's token span; frame mean = midpoint of
    the frame. Exercises head offsets, frame offsets, ragged last blocks and a
    KV head stride larger than the used length.
    """
    B, H, D, F, bt, NF, n_cur = 2, 2, 3, 10, 4, 3, 2
    stride = NF * F + 5
    s = oracle.Shape(B, H, D, F, bt, NF, 0, 0, n_cur, kv_stride=stride)
    k = torch.zeros(B, H, stride, D)
    q = torch.zeros(B, H, n_cur * F, D)
    for b in range(B):
        for h in range(H):
            off = 40 * (b * H + h)
            for d in range(D):
                k[b, h, :, d] = torch.arange(stride) + off + 3 * d
                q[b, h, :, d] = torch.arange(n_cur * F) + off + 3 * d + 1
    assert k.max() < 256  # integers below 256 are exact in bf16
    qp, kp, kf = oracle.pool(s, q.to(torch.bfloat16), k.to(torch.bfloat16))
    bpf = s.bpf
    for b in range(B):
        for h in range(H):
            off = 40 * (b * H + h)
            for tau in range(NF):
                for j in range(bpf):
                    t0, t1 = tau * F + j * bt, tau * F + min((j + 1) * bt, F)
                    mid = (t0 + t1 - 1) / 2
                    np.testing.assert_allclose(kp[b, h, tau * bpf + j], mid + off + 3 * np.arange(D), atol=1e-12)
                np.testing.assert_allclose(kf[b, h, tau], tau * F + (F - 1) / 2 + off + 3 * np.arange(D), atol=1e-12)
            for f in range(n_cur):
                for j in range(bpf):
                    t0, t1 = f * F + j * bt, f * F + min((j + 1) * bt, F)
                    mid = (t0 + t1 - 1) / 2
                    np.testing.assert_allclose(qp[b, h, f * bpf + j], mid + off + 1 + 3 * np.arange(D), atol=1e-12)


def test_pool_constant_and_frame_identity():
    """Constant tokens pool to the constant; the frame mean equals the
    token-count-weighted mean of the frame's block means (computed here from
    the block means, while the oracle sums the frame's tokens directly)."""
    g = torch.Generator().manual_seed(7)
    B, H, D, F, bt, NF, n_cur = 1, 3, 8, 150, 64, 4, 1
    s = oracle.Shape(B, H, D, F, bt, NF, 1, 1, n_cur)
    k = torch.randn(B, H, NF * F, D, generator=g).to(torch.bfloat16)
    q = torch.full((B, H, n_cur * F, D), 0.75).to(torch.bfloat16)
    qp, kp, kf = oracle.pool(s, q, k)
    np.testing.assert_array_equal(qp, 0.75)
    bpf = s.bpf
    counts = np.array([min((j + 1) * bt, F) - j * bt for j in range(bpf)], np.float64)
    for tau in range(NF):
        blocks = kp[:, :, tau * bpf:(tau + 1) * bpf, :]
        from_blocks = (blocks * counts[None, None, :, None]).sum(2) / F
        np.testing.assert_allclose(kf[:, :, tau], from_blocks, rtol=1e-13, atol=1e-14)
    # Mean of the whole frame, taken by a library routine on the fp64 tokens.
    kt = k.double().numpy().reshape(B, H, NF, F, D)
    np.testing.assert_allclose(kf, kt.mean(axis=3), rtol=1e-13, atol=1e-14)
