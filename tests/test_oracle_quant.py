"""Pins of the oracle's FP4 quantisation, ratio-2 pairing and block pooling (no GPU).

The quantiser is pinned by closed forms and invariants that a plausible slip
would break: exact round trips of representable rows, the error bound implied
by E4M3 scale rounding, sign symmetry, power-of-two scaling, idempotence, the
nibble order, the zero-scale rule, and the scale as torch's own E4M3 cast of
amax/6.
"""
import numpy as np
import torch

import synth

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _codes_unpacked(codes):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def _rows(n, seed=0):
    return synth.kv_rows(1001, seed, 0, n)


def test_scale_is_e4m3_of_amax_over_6(orc):
    x = _rows(512)
    _, scales = orc.quant_rows(x)
    amax = np.abs(x.reshape(-1, 16, 16)).max(axis=2).astype(np.float32)
    t = (amax / np.float32(6.0)).astype(np.float32)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(scales, ref)


def test_roundtrip_error_bound(orc):
    x = _rows(2048, seed=1)
    codes, scales = orc.quant_rows(x)
    xh = orc.dequant(codes, scales)
    s = np.array([[orc.e4m3_value(b) for b in row] for row in scales[:256]])
    err = np.abs(x[:256].astype(np.float64) - xh[:256]).reshape(256, 16, 16)
    # nearest rounding on the E2M1 grid: error <= half the local spacing (<= s),
    # and saturation beyond 6s is at most 0.4 s since s >= (amax/6)(1 - 2^-4)
    assert np.all(err <= s[:, :, None] * 1.0 + 1e-30)
    y = np.abs(x[:256].astype(np.float64)).reshape(256, 16, 16) / s[:, :, None]
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * s[:, :, None]
    sat = np.maximum(np.abs(x[:256]).reshape(256, 16, 16) - 6 * s[:, :, None], 0)
    assert np.all(err <= np.maximum(half_step, sat) + 1e-12)
    assert np.all(sat <= 0.4 * s[:, :, None] + 1e-12)


def test_exact_representable_row(orc):
    # a block whose amax is 6 gets scale 1.0 (0x38); grid values survive exactly
    vals = np.array([6, -6, 0.5, -0.5, 1, 1.5, 2, 3, 4, -4, 0, -0.0, 1.5, -3, 2, 6], np.float32)
    x = np.tile(vals, 16)[None, :] * np.repeat(2.0 ** np.arange(-7, 9), 16)[None, :].astype(np.float32)
    codes, scales = orc.quant_rows(x)
    for b in range(16):
        assert orc.e4m3_value(scales[0, b]) == 2.0 ** (b - 7)
    np.testing.assert_array_equal(orc.dequant(codes, scales)[0], x[0].astype(np.float64))


def test_nibble_order_and_sign_of_zero(orc):
    x = np.zeros((1, 256), np.float32)
    x[0, 6] = 6.0      # channel 6 -> low nibble of byte 3
    x[0, 9] = -3.0     # channel 9 -> high nibble of byte 4
    x[0, 7] = -0.01    # rounds to zero, keeps its sign: code 0x8 (high nibble of byte 3)
    codes, scales = orc.quant_rows(x)
    assert scales[0, 0] == 0x38  # amax 6 -> scale 1.0
    assert codes[0, 3] == (0x7 | (0x8 << 4))
    assert codes[0, 4] == (0xD << 4)
    assert np.count_nonzero(codes[0]) == 2


def test_zero_and_tiny_blocks(orc):
    x = np.zeros((3, 256), np.float32)
    x[1, :16] = -0.0
    x[2, :16] = 5.0 * 2.0 ** -10 * np.sign(np.arange(16) - 7.5)  # amax/6 < 2^-10 -> scale 0
    codes, scales = orc.quant_rows(x)
    assert not scales.any() and not codes.any()


def test_sign_symmetry(orc):
    x = _rows(256, seed=2)
    c1, s1 = orc.quant_rows(x)
    c2, s2 = orc.quant_rows(-x)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1 ^ 0x88, c2)


def test_power_of_two_scaling(orc):
    x = _rows(256, seed=3)
    c1, s1 = orc.quant_rows(x)
    c2, s2 = orc.quant_rows(x * np.float32(4.0))
    ok = (s1 >= 0x08) & (s1 <= 0x6F)  # normal scales that stay normal and finite when x4
    np.testing.assert_array_equal(s2[ok], s1[ok] + 0x10)
    u1, u2 = _codes_unpacked(c1).reshape(-1, 16, 16), _codes_unpacked(c2).reshape(-1, 16, 16)
    np.testing.assert_array_equal(u1[ok], u2[ok])


def test_idempotent(orc):
    x = _rows(512, seed=4)
    c1, s1 = orc.quant_rows(x)
    xh = orc.dequant(c1, s1).astype(np.float32)
    c2, s2 = orc.quant_rows(xh)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1, c2)


def test_ratio2_pair_mean(orc):
    x = _rows(256, seed=5)
    dup = np.repeat(x, 2, axis=0)
    c1, s1 = orc.quant_rows(x)
    c2, s2 = orc.quant_rows(dup, ratio=2)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)
    opp = np.stack([x, -x], axis=1).reshape(-1, 256)  # pairs cancel: zero entries
    c3, s3 = orc.quant_rows(opp, ratio=2)
    assert not c3.any() and not s3.any()
    # a pair (a, b) equals the entry of (a + b) / 2 computed in fp32
    pair = x[:200].reshape(100, 2, 256)
    c4, s4 = orc.quant_rows(pair.reshape(200, 256), ratio=2)
    m = ((pair[:, 0] + pair[:, 1]) * np.float32(0.5)).astype(np.float32)
    c5, s5 = orc.quant_rows(m)
    np.testing.assert_array_equal(c4, c5)
    np.testing.assert_array_equal(s4, s5)


def test_pooling(orc):
    k = synth.idx_k_rows(1001, 0, 0, 8 * 50 + 3)  # 50 full blocks + one block of 3
    pooled = orc.pool_blocks(k)
    assert pooled.shape == (51, 64)
    kf = orc.bf16_to_f32(k).reshape(-1, 64).astype(np.float64)
    mean = np.stack([kf[8 * j:min(8 * j + 8, kf.shape[0])].mean(axis=0) for j in range(51)])
    got = orc.bf16_to_f32(pooled).reshape(51, 64).astype(np.float64)
    # bf16 rounding (2^-9 relative) plus fp32 summation error of <= 8 terms
    bound = np.abs(mean) * 2.0 ** -8 + 8 * 2.0 ** -24 * np.abs(kf).max() + 1e-30
    assert np.all(np.abs(got - mean) <= bound)
    # identical rows pool to themselves (full and partial blocks)
    same = np.repeat(k[:3], 8, axis=0)[:19]
    np.testing.assert_array_equal(orc.pool_blocks(np.repeat(k[:1], 19, axis=0)), np.repeat(k[:1], 3, axis=0))
    assert orc.pool_blocks(same).shape == (3, 64)
    # the last partial block averages only the rows present (n = 3): rows a, a, -a -> a/3
    a = synth.to_bf16_bits(np.full((1, 64), 3.0, np.float32))
    na = synth.to_bf16_bits(np.full((1, 64), -3.0, np.float32))
    p = orc.pool_blocks(np.concatenate([a, a, na]))
    assert np.all(orc.bf16_to_f32(p) == 1.0)
