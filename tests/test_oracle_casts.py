"""Pins for the oracle's half-format casts: torch's CPU casts are the library
routine these must reduce to (round-to-nearest-even, gradual underflow,
overflow to infinity)."""

import numpy as np
import pytest
import torch

import oracle as O

TORCH = {O.BF16: torch.bfloat16, O.FP16: torch.float16}


def torch_encode(f32: np.ndarray, dtype: int) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(f32, np.float32)).to(TORCH[dtype])
    return t.view(torch.int16).numpy().view(np.uint16)


def torch_decode(h: np.ndarray, dtype: int) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(h, np.uint16).view(np.int16)).view(TORCH[dtype])
    return t.to(torch.float32).numpy()


def assert_same_encoding(bits_f32: np.ndarray, dtype: int):
    f = bits_f32.view(np.float32)
    a = O.float_to_half(f, dtype)
    b = torch_encode(f, dtype)
    nan = np.isnan(f)
    # NaN payloads are not part of the contract; NaN must stay NaN
    assert np.array_equal(a[~nan], b[~nan]), f"first mismatch at {np.flatnonzero(a[~nan] != b[~nan])[:5]}"
    back = O.half_to_float(a[nan], dtype)
    assert np.all(np.isnan(back))


@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_decode_all_65536(dtype):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    a = O.half_to_float(h, dtype)
    b = torch_decode(h, dtype)
    nan = np.isnan(b)
    assert np.array_equal(np.isnan(a), nan)
    assert np.array_equal(a[~nan].view(np.uint32), b[~nan].view(np.uint32))


def test_encode_bf16_every_high_half_at_rounding_boundaries():
    # bf16 keeps the top 16 bits of a float; the rounding decision depends on
    # the low 16 bits. Every high half is paired with the boundary patterns
    # (zero, just above zero, just below / at / just above the halfway point,
    # all ones) and a few random ones.
    rng = np.random.default_rng(7)
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000]
                    + rng.integers(0, 1 << 16, 8).tolist(), np.uint32)
    highs = np.arange(1 << 16, dtype=np.uint32)
    bits = (highs[:, None] << 16 | lows[None, :]).ravel()
    assert_same_encoding(bits, O.BF16)


def test_encode_fp16_every_exponent_and_top_mantissa_at_rounding_boundaries():
    # For fp16 the rounding point moves with the exponent (13 dropped bits for
    # normal results, more for subnormal results). All signs, exponents and
    # top 11 mantissa bits are enumerated, so every rounding point's halfway
    # pattern appears; the low 12 bits take boundary patterns.
    rng = np.random.default_rng(11)
    lows = np.array([0x000, 0x001, 0x7FF, 0x800, 0x801, 0xFFF]
                    + rng.integers(0, 1 << 12, 2).tolist(), np.uint32)
    tops = np.arange(1 << 20, dtype=np.uint32)  # sign(1) exponent(8) mantissa top(11)
    bits = (tops[:, None] << 12 | lows[None, :]).ravel()
    assert_same_encoding(bits, O.FP16)


def test_encode_named_values():
    cases = {
        O.FP16: [(65504.0, 0x7BFF), (65519.99, 0x7BFF), (65520.0, 0x7C00), (-65520.0, 0xFC00),
                 (2.0 ** -24, 0x0001), (2.0 ** -25, 0x0000), (1.5 * 2.0 ** -25, 0x0001),
                 (2.0 ** -14, 0x0400), (1.0, 0x3C00), (-0.0, 0x8000)],
        O.BF16: [(1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80), (1.0 + 3 * 2.0 ** -8, 0x3F82),
                 (3.4028234663852886e38, 0x7F80), (-2.0, 0xC000)],
    }
    for dtype, pairs in cases.items():
        f = np.array([p[0] for p in pairs], np.float32)
        want = np.array([p[1] for p in pairs], np.uint16)
        assert np.array_equal(O.float_to_half(f, dtype), want), (dtype, O.float_to_half(f, dtype))


@pytest.mark.slow
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_encode_exhaustive_2pow32(dtype):
    chunk = 1 << 26
    for start in range(0, 1 << 32, chunk):
        bits = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32)
        assert_same_encoding(bits, dtype)
