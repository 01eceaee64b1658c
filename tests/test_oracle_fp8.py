"""Pins of the oracle's FP8 frozen-weight format (CPU).

The pages name FP8 as a kernel family and a weight format ("Unsloth 深度分析报告",
关键设计决策; "Unsloth 还是 AirLLM", 核心原理) without defining it.  The reading:
OCP FP8 E4M3 codes, one fp32 scale per 64 input-dimension elements,
w = bf16_rne(fp32(e4m3) * scale).  The decode is pinned to torch's own
float8_e4m3fn type and to hand-computed codes; the dequantisation to an
independent evaluation (the exact product in float64, rounded once to fp32 and
once to bf16 by torch); planted mistakes must fail those pins."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_mlp_b200 import inputs as synth

ALL = np.arange(256, dtype=np.uint8)


def torch_e4m3(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def same(a, b):
    """Equal values, NaN where the other is NaN, and equal signs of zeros."""
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    nan = np.isnan(a)
    return (np.array_equal(nan, np.isnan(b)) and np.array_equal(a[~nan], b[~nan])
            and np.array_equal(np.signbit(a[~nan]), np.signbit(b[~nan])))


def test_decode_matches_torch_float8_for_every_code():
    assert same(oracle.e4m3_to_f64(ALL), torch_e4m3(ALL))


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0),
    (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),        # subnormals: m/8 * 2^-6
    (0x08, 2.0 ** -6),                               # smallest normal
    (0x38, 1.0), (0x3F, 1.875), (0xB8, -1.0),
    (0x7E, 448.0), (0xFE, -448.0),                   # largest finite
])
def test_decode_hand_computed(code, value):
    got = oracle.e4m3_to_f64(np.array([code], dtype=np.uint8))[0]
    assert got == value and np.signbit(got) == np.signbit(value)


def test_nan_codes():
    v = oracle.e4m3_to_f64(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.all(np.isnan(v))
    assert np.sum(np.isnan(oracle.e4m3_to_f64(ALL))) == 2


def independent_dequant(codes, scales):
    """exact product in float64 (<= 4 x 24 significant bits), rounded to fp32
    and then to bf16 by torch's conversions."""
    v = torch_e4m3(codes)
    s = np.repeat(np.asarray(scales, dtype=np.float32).astype(np.float64), 64, axis=1)
    with np.errstate(invalid="ignore", over="ignore"):
        prod = v * s
    t = torch.from_numpy(prod).to(torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def scale_set():
    rng = np.random.default_rng(7)
    sc = list(rng.uniform(-3, 3, 120).astype(np.float32)) + list(
        (10.0 ** rng.uniform(-44, 38, 120)).astype(np.float32))
    sc += [0.0, -0.0, 1e-45, -1e-45, 1e-40, 2.0 ** -126, 1.0, -1.0, 3.4e38, -3.4e38, 1 / 448, 0.1]
    return np.array(sc, dtype=np.float32)


def check_dequant(fn):
    sc = scale_set()
    rows = len(sc)
    codes = np.tile(ALL, (rows, 1))                              # [rows, 256]: 4 blocks of 64
    scales = np.repeat(sc[:, None], 4, axis=1)
    got = fn(codes, scales)
    ref = independent_dequant(codes, scales)
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    return same(f(got), f(ref))


def test_dequant_matches_independent_rounding():
    assert check_dequant(oracle.dequant_fp8)
    # specials: inf scale gives +-inf (NaN for a zero code), NaN codes give NaN
    codes = np.tile(ALL, (1, 1))
    got = oracle.dequant_fp8(codes, np.full((1, 4), np.inf, np.float32))
    v = (got.astype(np.uint32) << 16).view(np.float32)[0]
    e = oracle.e4m3_to_f64(ALL)
    assert np.all(np.isnan(v[(e == 0) | np.isnan(e)]))
    assert np.all(np.isinf(v[(e != 0) & ~np.isnan(e)]))


# planted mistakes: each must fail the pins above

def _decode_bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -7, (1 + m / 8.0) * np.exp2(e - 8.0))
    return np.where(c & 0x80, -1.0, 1.0) * np.where((e == 15) & (m == 7), np.nan, mag)


def _decode_no_subnormals(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 7
    mag = (1 + m / 8.0) * np.exp2(e - 7.0)
    return np.where(c & 0x80, -1.0, 1.0) * np.where((e == 15) & (m == 7), np.nan, mag)


@pytest.mark.parametrize("bad", [_decode_bias8, _decode_no_subnormals])
def test_planted_decode_mistakes_are_caught(bad):
    assert not same(bad(ALL), torch_e4m3(ALL))


def test_planted_rounding_mistake_is_caught():
    def scale_in_bf16(codes, scales):       # rounds the scale to bf16 before the product
        s16 = oracle.f32_to_bf16_rne(np.asarray(scales, np.float32))
        s = (s16.astype(np.uint32) << 16).view(np.float32)
        return oracle.dequant_fp8(codes, s)
    assert not check_dequant(scale_in_bf16)


def test_quantiser_round_trip():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((96, 448)).astype(np.float32) * np.float32(0.02)
    w[4, 64:128] = 0.0
    codes, scales = synth.quantize_fp8(w)
    assert codes.dtype == np.uint8 and scales.dtype == np.float32 and scales.shape == (96, 7)
    back = oracle.bf16_to_f64(oracle.dequant_fp8(codes, scales))
    amax = np.repeat(np.abs(w.reshape(96, 7, 64)).max(axis=2), 64, axis=1)
    # E4M3 keeps 3 mantissa bits (relative half-ulp 2^-4 for normals; subnormals
    # absolute 2^-10 of the block max); bf16 adds 2^-9
    err = np.abs(back - w)
    assert np.all(err <= 2.0 ** -4 * np.abs(w) * 1.01 + amax * 2.0 ** -10 / 448 * 2 + 2.0 ** -9 * np.abs(w))
    assert np.all(back[4, 64:128] == 0.0)
