"""Pins for the oracle's number formats (E2M1, E8M0, E4M3, BF16) against the
published format tables and independent library implementations."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
from tests._golden import e2m1_table, e4m3_points, e8m0_points, kv


def test_e2m1_all_codes_match_table():
    tab = e2m1_table()
    for c in range(16):
        got = oracle.e2m1(c)
        assert got == tab[c], c
        assert math.copysign(1.0, got) == math.copysign(1.0, tab[c]), c  # -0 for code 8


def test_e8m0_landmarks_and_doubling():
    for e, v in e8m0_points():
        got = oracle.e8m0(e)
        if math.isnan(v):
            assert math.isnan(got)
        else:
            assert got == v, e
    for e in range(0, 254):
        assert oracle.e8m0(e + 1) == 2.0 * oracle.e8m0(e)


def test_e4m3_landmarks():
    for c, v in e4m3_points():
        got = oracle.e4m3(c)
        if math.isnan(v):
            assert math.isnan(got), hex(c)
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v), hex(c)


def test_e4m3_all_codes_match_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], c


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(1)
    bits = np.concatenate([rng.integers(0, 1 << 16, 4000), [0, 0x8000, 0x0001, 0x7F7F, 0xFF7F, 0x3F80]])
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for b, r in zip(bits, ref):
        got = oracle.bf16_value(int(b))
        assert (math.isnan(got) and math.isnan(r)) or got == r


def test_bf16_rne_matches_torch_on_fp32_inputs():
    # fp32 -> bf16 in torch is one RNE rounding; on fp32-representable inputs the
    # oracle's direct fp64 rounding must agree bit for bit.
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        rng.standard_normal(3000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-38).astype(np.float32),
        (rng.standard_normal(1000) * 1e30).astype(np.float32),
    ])
    # exact midpoints between adjacent bf16 values: ties go to the even significand
    base = torch.from_numpy(rng.integers(0x0080, 0x7F00, 500).astype(np.int16)).view(torch.bfloat16)
    mids = (base.to(torch.float32).view(torch.int32) + (1 << 15)).view(torch.float32).numpy()
    vals = np.concatenate([vals, mids, -mids])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, r in zip(vals, ref):
        assert oracle.bf16_rne(float(v)) == int(r), v


def test_e4m3_encode_matches_torch_rne_in_range():
    vals = []
    finite = [oracle.e4m3(c) for c in range(0x7F)]  # 0 .. 448 ascending
    for lo, hi in zip(finite[:-1], finite[1:]):
        mid = np.float32((lo + hi) / 2)  # exact in fp32
        vals += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)), np.float32(lo)]
    rng = np.random.default_rng(3)
    vals += list((rng.standard_normal(3000) * 40).astype(np.float32))
    vals += list((rng.standard_normal(1000) * 1e-2).astype(np.float32))
    vals += [np.float32(464.0), np.float32(448.0), np.float32(449.0)]
    v = np.array(vals, np.float32)
    v = np.concatenate([v, -v])
    v = v[np.abs(v) <= 464.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(v, ref):
        assert oracle.e4m3_encode(float(x)) == int(r), float(x)


def test_e4m3_encode_saturates():
    for v, code in [(465.0, 0x7E), (480.0, 0x7E), (1e6, 0x7E), (float("inf"), 0x7E),
                    (-465.0, 0xFE), (-1e30, 0xFE), (float("-inf"), 0xFE)]:
        assert oracle.e4m3_encode(v) == code, v
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    assert oracle.e4m3_encode(-1e-30) == 0x80  # rounds to zero, keeps its sign


def test_lm_head_fp8_bytes_are_half_of_bf16():
    g = kv("lm_head_bytes.txt")
    V, H = g["vocab"], g["hidden"]
    assert V * H * np.dtype(np.uint8).itemsize == g["fp8_code_bytes"]
    assert V * H * 2 == g["bf16_bytes"]
    assert 2 * g["fp8_code_bytes"] == g["bf16_bytes"]
