"""Pins for the oracle's number formats: decoding and RNE encoding of bf16 and
fp16, the binary32 add that forms x = x1 + x2, and round-half-to-even.

Each is checked against an independent library implementation of the same
IEEE / bfloat16 definition (torch's bfloat16, numpy's float16, numpy.rint),
exhaustively over all 2^16 patterns where that is possible and on every tie.
"""
import numpy as np
import pytest
import torch

import oracle

ALL16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def _torch_bf16_bits(f32):
    return torch.from_numpy(np.ascontiguousarray(f32, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _numpy_fp16_bits(f32):
    with np.errstate(over="ignore"):
        return np.ascontiguousarray(f32, np.float32).astype(np.float16).view(np.uint16)


def _same_values(got, ref):
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_decode_bf16_every_pattern():
    ref = torch.from_numpy(ALL16.view(np.int16)).view(torch.bfloat16).double().numpy()
    _same_values(oracle.decode16(ALL16, "bf16"), ref)


def test_decode_fp16_every_pattern():
    ref = ALL16.view(np.float16).astype(np.float64)
    _same_values(oracle.decode16(ALL16, "fp16"), ref)


def _finite_random_f32(rng, count):
    bits = rng.integers(0, 2 ** 32, count, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    return f[np.isfinite(f)]


def _fp16_range_f32(rng, count):
    # magnitudes spread over binary16's whole range, subnormals and overflow included
    e = rng.uniform(-27.0, 17.0, count)
    s = rng.choice([-1.0, 1.0], count)
    return (s * np.exp2(e)).astype(np.float32)


def test_encode_bf16_random_and_specials():
    rng = np.random.default_rng(123)
    f = np.concatenate([
        _finite_random_f32(rng, 400_000),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38, 3.4028235e38,
                  1e-45, -1e-45, 1.1754942e-38, 1.0, -1.0], np.float32)])
    assert np.array_equal(oracle.encode16(f, "bf16"), _torch_bf16_bits(f))


def test_encode_bf16_every_tie_and_neighbours():
    hi = ALL16.astype(np.uint32) << 16
    for low in (0x7FFF, 0x8000, 0x8001):
        f = (hi | low).view(np.float32)
        f = f[np.isfinite(f)]
        assert np.array_equal(oracle.encode16(f, "bf16"), _torch_bf16_bits(f)), hex(low)


def test_encode_fp16_random_and_specials():
    rng = np.random.default_rng(7)
    f = np.concatenate([
        _fp16_range_f32(rng, 400_000), _finite_random_f32(rng, 100_000),
        np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.996, 65520.0, -65520.0,
                  2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -14, 1.0], np.float32)])
    assert np.array_equal(oracle.encode16(f, "fp16"), _numpy_fp16_bits(f))


def test_encode_fp16_every_tie():
    # exact midpoints between consecutive finite binary16 values (and between
    # the largest finite value and 2^16); each is exact in binary32
    pos = np.arange(0, 0x7C00, dtype=np.uint16)
    v = pos.view(np.float16).astype(np.float64)
    nxt = np.append(v[1:], 65536.0)
    mid = ((v + nxt) / 2.0)
    f = mid.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), mid)  # exact
    f = np.concatenate([f, -f])
    assert np.array_equal(oracle.encode16(f, "fp16"), _numpy_fp16_bits(f))


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_add_round_matches_binary32_add(dtype):
    rng = np.random.default_rng(11)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    a = rng.integers(0, 65536, 300_000).astype(np.uint16)
    b = rng.integers(0, 65536, 300_000).astype(np.uint16)
    # nearby magnitudes (cancellation) and wide exponent gaps
    b[:50_000] = a[:50_000] ^ 0x8000
    b[50_000:100_000] = (a[50_000:100_000] ^ 0x8000) + 1
    ta = torch.from_numpy(a.view(np.int16)).view(tdt).float()
    tb = torch.from_numpy(b.view(np.int16)).view(tdt).float()
    ok = (torch.isfinite(ta) & torch.isfinite(tb)).numpy()
    s = (ta + tb)  # IEEE binary32 add on the CPU
    ref = s.to(tdt).view(torch.int16).numpy().view(np.uint16)
    got = oracle.add_round(a, b, dtype)
    fin = ok & np.isfinite(s.numpy())
    assert np.array_equal(got[fin], ref[fin])


def test_add_round_cancellation_gives_positive_zero():
    one = np.array([0x3F80], np.uint16)
    m_one = np.array([0xBF80], np.uint16)
    assert oracle.add_round(one, m_one, "bf16")[0] == 0x0000


def test_round_half_even():
    vals = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.5, -127.5, 3.4999999999, 3.5000000001,
            0.49999999999999994, 1e15 + 0.5, -7.5, 6.5]
    for v in vals:
        assert oracle.round_half_even(v) == np.rint(v), v
