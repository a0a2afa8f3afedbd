"""Pins of the oracle's number formats (no GPU).

E2M1 / E4M3 / bf16 encoders are checked against the textbook tables in
tests/golden/number_formats.json, against brute-force nearest-value search and
against torch's own float8_e4m3fn / bfloat16 casts.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def brute_e2m1(y: np.ndarray) -> np.ndarray:
    """Nearest E2M1 magnitude by exhaustive search; ties to the even code."""
    # beyond 6 the nearest magnitude is 6; clamping keeps fp64 distances exact
    a = np.minimum(np.abs(y.astype(np.float64)), 7.0)
    dist = np.abs(a[:, None] - E2M1_MAG[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among tied codes pick the even one (there are at most two, adjacent)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)
    return code | (np.signbit(y).astype(np.uint8) << 3)


def test_e2m1_table(orc):
    vals = _golden("number_formats.json")["e2m1_values"]
    for c in range(16):
        v = orc.e2m1_value(c)
        assert v == vals[c] and math.copysign(1, v) == math.copysign(1, vals[c])
        # every code re-encodes to itself (sign of zero included)
        assert orc.e2m1_encode(np.float32(v))[0] == c


def test_e2m1_encoder_vs_brute_force(orc):
    f32 = np.float32
    pts = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 2.0, 4.0, 1.0, 0.5]
    chunks = []
    for p in pts:  # 4096 consecutive fp32 values around every rounding boundary
        u = np.array([f32(p)]).view(np.uint32)[0]
        chunks.append(np.arange(u - 2048, u + 2048, dtype=np.uint32).view(np.float32))
    rng = np.random.default_rng(7)
    chunks.append(rng.uniform(-8, 8, 1_000_000).astype(np.float32))
    chunks.append(np.array([0.0, -0.0, 1e-30, -1e-30, 1e30, -1e30, 6.4, -6.4, 7.0, 1e-45], np.float32))
    y = np.concatenate(chunks)
    y = np.concatenate([y, -y])
    np.testing.assert_array_equal(orc.e2m1_encode(y), brute_e2m1(y))


def test_e2m1_ties_explicit(orc):
    # ties go to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2, 2.5->2, 3.5->4, 5->4
    y = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 100.0, -0.2], np.float32)
    assert orc.e2m1_encode(y).tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 8]


def test_e4m3_table_vs_golden_and_torch(orc):
    spec = _golden("number_formats.json")["e4m3_special"]
    for k, v in spec.items():
        got = orc.e4m3_value(int(k, 16))
        if v == "nan":
            assert math.isnan(got)
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v)
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = codes.to(torch.float64).numpy()
    for c in range(256):
        got = orc.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c], hex(c)


def test_e4m3_encoder_exhaustive_vs_torch(orc):
    """Every non-negative fp32 below 464 (all values that round into range)."""
    top = np.array([464.0], np.float32).view(np.uint32)[0]
    step = 1 << 24
    for lo in range(0, int(top), step):
        u = np.arange(lo, min(lo + step, int(top)), dtype=np.uint32)
        x = u.view(np.float32)
        ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = orc.e4m3_encode(x)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_encoder_negative_and_saturation(orc):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-460, 0, 2_000_000), -rng.uniform(0, 1e-2, 200_000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(orc.e4m3_encode(x), ref)
    # saturating finite: everything at or beyond 448 maps to +-448
    big = np.array([448.0, 463.9, 464.0, 480.0, 1e6, np.inf], np.float32)
    assert set(orc.e4m3_encode(big).tolist()) == {0x7E}
    assert set(orc.e4m3_encode(-big).tolist()) == {0xFE}


def test_bf16_rne_vs_torch(orc):
    rng = np.random.default_rng(11)
    hi = rng.integers(0, 1 << 16, 64, dtype=np.uint32)
    lo = np.arange(1 << 16, dtype=np.uint32)
    u = ((hi[:, None] << 16) | lo[None, :]).ravel()  # every low half for 64 high halves
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.f32_to_bf16(x), ref)
    np.testing.assert_array_equal(orc.bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(
        torch.bfloat16).to(torch.float32).numpy())
