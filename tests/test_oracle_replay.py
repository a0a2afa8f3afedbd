"""Pins of the oracle's SWA Bounded Replay (no GPU): closed forms that a
dropped term, a transposed operand or a wrong rounding would break."""
import numpy as np

import synth


def bf(x):
    return synth.to_bf16_bits(np.asarray(x, np.float32))


def test_identity_projection_reproduces_the_rows(orc):
    # d = 256 and W = I: every replayed row is the hidden state itself
    h = synth.swa_rows(1001, 0, 0, 128)
    w = bf(np.eye(256, dtype=np.float32))
    np.testing.assert_array_equal(orc.swa_replay(h, w), h)


def test_scaled_permutation(orc):
    # W = 2 P: out[t][c] = 2 h[t][perm[c]], exact in bf16 (a power of two)
    rng = np.random.default_rng(1)
    d = 320
    perm = rng.permutation(d)[:256]
    w = np.zeros((256, d), np.float32)
    w[np.arange(256), perm] = 2.0
    h = synth.hidden_rows(1001, 0, 0, 17, d)
    got = orc.swa_replay(h, bf(w))
    want = bf(2.0 * orc.bf16_to_f32(h)[:, perm])
    np.testing.assert_array_equal(got, want)


def test_unit_hidden_state_selects_a_weight_column(orc):
    d = 128
    w = synth.kv_projection(1001, 3, d)
    h = np.zeros((d, d), np.float32)
    h[np.arange(d), np.arange(d)] = 1.0
    got = orc.swa_replay(bf(h), w)          # row t = column t of W
    np.testing.assert_array_equal(got, w.T)


def test_against_fp64_matmul_rounded(orc):
    # the definition written out: fp64 sums rounded to fp32, then to bf16
    d = 192
    h = synth.hidden_rows(1001, 1, 2, 40, d)
    w = synth.kv_projection(1001, 1, d)
    ref = orc.bf16_to_f32(h).astype(np.float64) @ orc.bf16_to_f32(w).astype(np.float64).T
    np.testing.assert_array_equal(orc.swa_replay(h, w), bf(ref.astype(np.float32)))
    # K channels come from rows 0..127 of W, V channels from rows 128..255
    w2 = w.copy()
    w2[128:] = 0
    out2 = orc.swa_replay(h, w2)
    assert (orc.bf16_to_f32(out2)[:, 128:] == 0).all()
    np.testing.assert_array_equal(out2[:, :128], orc.swa_replay(h, w)[:, :128])


def test_replayed_rows_have_the_window_distribution(orc):
    h = synth.hidden_rows(1004, 0, 0, 128)
    w = synth.kv_projection(1004, 0)
    x = orc.bf16_to_f32(orc.swa_replay(h, w)).astype(np.float64)
    g = synth.gain(1004).astype(np.float64)
    # per-channel standard deviation close to the gain (N(0,1) x gain)
    assert np.allclose(x.std(axis=0) / g, 1.0, atol=0.25)
