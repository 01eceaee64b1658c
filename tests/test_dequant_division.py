"""The int4 dequantisation kernel divides by 7 without a divide instruction:
with r = fl32(1/7) and x = q * scale (exact), it evaluates, two lanes at a
time and from -x so that a zero keeps its sign,

    y = (-x) * (-r)          (rounded to fp32)
    e = 7 * y + (-x)         (one FMA: the exact residual, negated)
    z = e * (-r) + y         (one FMA)

This test replays that sequence in numpy, rounding exactly where the GPU
rounds, and checks it bit for bit against IEEE fp32 division x / 7 for
every int4 code (-8..7) and every finite fp16 scale (positive, negative,
+-0, subnormal): the claim the kernel's correctness rests on.  (The GPU
tests compare the kernel's output with the oracle bit for bit on a sample of
scales; this covers all of them.)"""
from fractions import Fraction

import numpy as np

R = np.float32(1.0) / np.float32(7.0)


def _round_sum_f32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """fl32(a + b) for float64 arrays whose products were exact: the float64
    sum is rounded once more to fp32, which can only differ from a single
    rounding when it lands within a few float64 ulps of an fp32 rounding
    boundary; those few cases are redone with exact rationals."""
    s64 = a + b
    out = s64.astype(np.float32)
    # distance of the float64 sum to the nearest fp32 midpoint, in float64 ulps
    lo = out.astype(np.float64)
    up = np.nextafter(out, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(out, np.float32(-np.inf)).astype(np.float64)
    mid = np.minimum(np.abs(s64 - (lo + up) / 2), np.abs(s64 - (lo + dn) / 2))
    risky = np.nonzero(mid <= 8 * np.spacing(np.abs(s64)) + 1e-300)[0]
    for i in risky:
        exact = Fraction(float(a[i])) + Fraction(float(b[i]))
        if exact == 0:
            continue  # zero results: the sign rule is that of the float64 sum, checked below
        c = np.float32(float(exact))
        cands = [c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))]
        best = min(cands, key=lambda v: (abs(Fraction(float(v)) - exact), int(np.float32(v).view(np.uint32)) & 1))
        out[i] = best
    return out


def test_fma_corrected_division_by_seven_is_ieee_for_every_code_and_scale():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    scales = bits.view(np.float16)
    scales = scales[np.isfinite(scales)].astype(np.float32)          # 63,488 finite fp16 values
    codes = np.arange(-8, 8, dtype=np.float32)
    q, s = np.meshgrid(codes, scales, indexing="ij")
    q, s = q.ravel(), s.ravel()
    x = q * s                                                          # exact in fp32
    ref = x / np.float32(7.0)                                          # IEEE correctly rounded

    neg_x = (q * -s).astype(np.float32)                                # q * (-scale), exact
    y = (neg_x.astype(np.float64) * float(-R)).astype(np.float32)      # product exact in f64, one rounding
    e = (y.astype(np.float64) * 7.0 + neg_x.astype(np.float64)).astype(np.float32)  # exact residual
    z = _round_sum_f32(e.astype(np.float64) * float(-R), y.astype(np.float64))
    # IEEE zero sums: +0 unless both addends are -0 (round to nearest)
    zero = (e.astype(np.float64) * float(-R) + y.astype(np.float64)) == 0
    both_neg = np.signbit(e * -R) & np.signbit(y)
    z[zero] = np.where(both_neg[zero], np.float32(-0.0), np.float32(0.0))

    mismatch = z.view(np.uint32) != ref.view(np.uint32)
    assert not mismatch.any(), (q[mismatch][:5], s[mismatch][:5], z[mismatch][:5], ref[mismatch][:5])
    assert len(z) == 16 * 63488


def test_the_plain_product_alone_is_not_enough():
    """Without the correction step the quotient is often one ulp off (the
    reason the kernel has it)."""
    s = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    x = np.float32(3.0) * s
    plain = (x.astype(np.float64) * float(R)).astype(np.float32)
    assert np.mean(plain.view(np.uint32) != (x / np.float32(7.0)).view(np.uint32)) > 0.3
