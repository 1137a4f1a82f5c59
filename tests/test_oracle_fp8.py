"""Pins for the oracle's FP8 (e4m3) inputs and its fp64-input attention.

Source: the pages quantise linear layers to FP8 with per-channel weight scales
and per-token activation scales (163.com article, deployment section;
gist.science results, "FP8 linear layers"); an FP8 attention is not described.
Readings: e4m3 with round-to-nearest-even and saturation at 448; Q and K
scaled per token, V per channel of each head; scale = max |x| / 448.
"""
import numpy as np
import pytest
import torch

import oracle


def _e4m3_table():
    """Every finite e4m3 value, from the library's own float8 type."""
    vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    vals = vals[torch.isfinite(vals)].double().numpy()
    return np.unique(vals)


def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).double().numpy()


def test_e4m3_matches_torch_on_values_midpoints_and_random():
    table = _e4m3_table()
    assert table.max() == 448.0 and table.min() == -448.0 and len(table) == 253  # +-0 merge
    np.testing.assert_array_equal(oracle.e4m3(table), table)
    pos = table[table >= 0]
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties in fp32
    for m in (mids, -mids):
        np.testing.assert_array_equal(oracle.e4m3(m), _torch_e4m3(m))
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-2 ** -5, 2 ** -5, 5000),
                        rng.standard_normal(5000)]).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.e4m3(x), _torch_e4m3(x))


def test_e4m3_saturates():
    np.testing.assert_array_equal(oracle.e4m3([448.0, 460.0, 500.0, 1e30, -1e30]),
                                  [448.0, 448.0, 448.0, 448.0, -448.0])


def test_quant_rows_hand_worked():
    x = torch.tensor([[1.0, 2.0, 3.0, 4.0], [-8.0, 0.5, 2.0, 1.0], [0.0, 0.0, 0.0, 0.0]],
                     dtype=torch.bfloat16)
    out, sc = oracle.quant_rows_e4m3(x)
    # row 0: s = 4/448, x/s = 112, 224, 336, 448; 336 lies halfway between 320 and 352 -> 320
    np.testing.assert_allclose(sc, [4 / 448, 8 / 448, 1.0], rtol=0, atol=0)
    np.testing.assert_allclose(out[0], [1.0, 2.0, 320 * 4 / 448, 4.0], rtol=1e-15)
    # row 1: s = 8/448, x/s = -448, 28, 112, 56, all e4m3 values
    np.testing.assert_allclose(out[1], [-8.0, 0.5, 2.0, 1.0], rtol=1e-15)
    np.testing.assert_array_equal(out[2], 0.0)


def test_quant_cols_hand_worked_per_head():
    x = torch.zeros(1, 2, 3, 2, dtype=torch.bfloat16)
    x[0, 0, :, 0] = torch.tensor([3.0, -6.0, 1.5])   # 224, -448, 112: exact
    x[0, 0, :, 1] = torch.tensor([1.0, 2.0, 3.0])    # 149.33.., 298.66.., 448
    x[0, 1, :, 0] = torch.tensor([0.25, 0.0, 0.0])   # a head of its own
    out, sc = oracle.quant_cols_e4m3(x)
    np.testing.assert_allclose(sc[0, 0], [6 / 448, 3 / 448])
    np.testing.assert_allclose(out[0, 0, :, 0], [3.0, -6.0, 1.5], rtol=1e-15)
    # 149.33 -> 144 (step 8 in [128, 256)), 298.67 -> 288 (step 32 in [256, 448])
    np.testing.assert_allclose(out[0, 0, :, 1], [144 * 3 / 448, 288 * 3 / 448, 3.0], rtol=1e-15)
    np.testing.assert_allclose(out[0, 1, :, 0], [0.25, 0.0, 0.0])
    assert sc[0, 1, 1] == 1.0  # an all-zero channel keeps scale 1


@pytest.mark.parametrize("seed", range(3))
def test_quant_keeps_the_largest_magnitude_and_the_error_bound(seed):
    rng = np.random.default_rng(seed)
    x = torch.tensor(rng.standard_normal((64, 32)) * 3, dtype=torch.bfloat16)
    xf = x.double().numpy()
    out, sc = oracle.quant_rows_e4m3(x)
    # the largest magnitude maps to 448 exactly, so it comes back up to the rounding of s * (x / s)
    np.testing.assert_allclose(np.abs(out).max(axis=1), np.abs(xf).max(axis=1), rtol=1e-15, atol=0)
    normal = np.abs(xf) / sc[:, None] >= 2 ** -6
    err = np.abs(out - xf)
    assert (err[normal] <= 2 ** -4 * np.abs(xf[normal]) * (1 + 1e-12)).all()
    assert (err[~normal] <= (2 ** -10 * sc[:, None] * np.ones_like(xf))[~normal] * (1 + 1e-12)).all()


def test_attention_f64_equals_attention_on_bf16_inputs():
    rng = np.random.default_rng(5)
    s = oracle.Shape(1, 2, 64, 100, 64, 5, 1, 1, 2, kv_stride=5 * 100 + 11)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 2, s.Lq, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, s.stride, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, s.stride, 64, generator=g).to(torch.bfloat16)
    cap = 4
    lst = np.sort(np.stack([rng.choice(s.Nkv, cap, replace=False) for _ in range(2 * s.Rq)]), axis=1)
    lst = lst.reshape(1, 2, s.Rq, cap).astype(np.int32)
    cnt = rng.integers(0, cap + 1, size=(1, 2, s.Rq)).astype(np.int32)
    a = oracle.attention(s, q, k, v, lst, cnt)
    b = oracle.attention_f64(s, q.double().numpy(), k.double().numpy(), v.double().numpy(), lst, cnt)
    np.testing.assert_array_equal(a, b)


def test_attention_on_fp8_inputs_stays_close():
    """A property, not a pin: quantising q, k and v (about 3.6 % rms rounding of each value)
    moves the output by a few percent of its size, neither zero (no quantisation) nor of its
    size (a missing scale)."""
    s = oracle.Shape(1, 1, 64, 128, 64, 4, 1, 1, 1)
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 1, s.Lq, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, s.stride, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 1, s.stride, 64, generator=g).to(torch.bfloat16)
    lst = np.tile(np.arange(s.Nkv, dtype=np.int32), (1, 1, s.Rq, 1))
    cnt = np.full((1, 1, s.Rq), s.Nkv, np.int32)
    ref = oracle.attention(s, q, k, v, lst, cnt)
    got = oracle.attention_fp8_inputs(s, q, k, v, lst, cnt)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 0.01 < rel < 0.08, rel


# ---- quantisation decided in fp32 (the precision the FP8 attention kernel uses) -----

def test_quant_rows_f32_hand_worked():
    """amax 3.5 gives the exact scale 3.5/448 = 2^-7, so every code is e4m3(128 x):
    0.30078125 (bf16 of 0.3) -> 38.5 -> 40 (step 4 in [32, 64)) -> 0.3125; a row whose
    amax is 448 keeps scale 1; an all-zero row gets scale 1 and zero codes."""
    x = torch.tensor([[3.5, -1.0, 0.3, 0.0],
                      [448.0, -20.0, 0.0107421875, 1.0],
                      [0.0, 0.0, 0.0, 0.0]]).to(torch.bfloat16)
    out, sc = oracle.quant_rows_e4m3_f32(x)
    assert sc.dtype == np.float32
    np.testing.assert_array_equal(sc, np.array([2.0 ** -7, 1.0, 1.0], np.float32))
    # row 1: -20 -> step 2 in [16, 32) -> -20; 0.0107421875 = 11 * 2^-10 -> subnormal step 2^-9 -> 5.5 * 2^-9
    # ties to even -> 6 * 2^-9 = 0.01171875
    np.testing.assert_array_equal(out, np.array([[3.5, -1.0, 0.3125, 0.0],
                                                 [448.0, -20.0, 0.01171875, 1.0],
                                                 [0.0, 0.0, 0.0, 0.0]]))


@pytest.mark.parametrize("seed", range(3))
def test_quant_rows_f32_matches_torch(seed):
    """Against torch: fp32 amax / 448 and fp32 division (IEEE, as C float arithmetic),
    then torch's float8_e4m3fn cast (round to nearest even) after clamping to +-448."""
    g = torch.Generator().manual_seed(100 + seed)
    mag = torch.exp(torch.randn(64, 1, generator=g) * 3.0)  # rows from ~1e-4 to ~1e4
    x = (torch.randn(64, 128, generator=g) * mag).to(torch.bfloat16)
    x[5] = 0.0
    out, sc = oracle.quant_rows_e4m3_f32(x)
    xf = x.float()
    amax = xf.abs().amax(-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    code = (xf / s[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).float()
    np.testing.assert_array_equal(sc, s.numpy())
    np.testing.assert_array_equal(out, s.double().numpy()[:, None] * code.double().numpy())


def test_quant_rows_f32_agrees_with_fp64_off_midpoints():
    """The fp32 and fp64 decisions differ only where x / s lies within fp32 rounding of an
    e4m3 midpoint: a handful of codes in 10^5, each one e4m3 step apart."""
    g = torch.Generator().manual_seed(7)
    x = torch.randn(1000, 128, generator=g).to(torch.bfloat16)
    a, sa = oracle.quant_rows_e4m3_f32(x)
    b, sb = oracle.quant_rows_e4m3(x)
    np.testing.assert_allclose(sa, sb, rtol=2 ** -23)
    ca, cb = a / sa.astype(np.float64)[:, None], b / sb[:, None]
    differ = np.abs(ca - cb) > 1e-9
    assert differ.sum() <= 40, differ.sum()
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(cb), 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(ca - cb)[differ] <= step[differ] * (1 + 1e-12))
