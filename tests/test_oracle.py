"""Pins for the fp64 CPU oracle: each test ties it to something other than
itself (finite differences, closed forms, a library SwiGLU MLP, exact rational
arithmetic, invariants of the LoRA parameterisation)."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_mlp_b200 import inputs as synth

ADAPTERS = ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")


def rand_params(rng, N, d, d_ff, r, scale_b=0.3):
    p = {
        "X": rng.standard_normal((N, d)),
        "Wg": rng.standard_normal((d_ff, d)) / math.sqrt(d),
        "Wu": rng.standard_normal((d_ff, d)) / math.sqrt(d),
        "Wd": rng.standard_normal((d, d_ff)) / math.sqrt(d_ff),
        "Ag": rng.uniform(-1, 1, (r, d)),
        "Bg": rng.standard_normal((d_ff, r)) * scale_b,
        "Au": rng.uniform(-1, 1, (r, d)),
        "Bu": rng.standard_normal((d_ff, r)) * scale_b,
        "Ad": rng.uniform(-1, 1, (r, d_ff)),
        "Bd": rng.standard_normal((d, r)) * scale_b,
    }
    dOut = rng.standard_normal((N, d))
    return p, dOut


def library_mlp(X, Wg, Wu, Wd):
    """Textbook SwiGLU MLP through torch's own silu (float64, CPU)."""
    F = torch.nn.functional
    return (F.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T


def relerr(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


# ----------------------------------------------------------------------------
# backward: central finite differences of L = <dOut, out>


@pytest.mark.parametrize("shape,alpha", [((3, 5, 7, 2), 3.0), ((4, 6, 10, 3), 1.5)])
def test_backward_matches_central_differences(shape, alpha):
    rng = np.random.default_rng(7)
    N, d, d_ff, r = shape
    p, dOut = rand_params(rng, N, d, d_ff, r)
    b = oracle.backward(p, alpha, dOut)
    eps = 1e-5

    def loss(q):
        return float(np.sum(dOut * oracle.forward(q, alpha)["out"]))

    for name, grad_name in [("X", "dX")] + [(a, "d" + a) for a in ADAPTERS]:
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(*p[name].shape):
            q = {k: v.copy() for k, v in p.items()}
            q[name][idx] += eps
            lp = loss(q)
            q[name][idx] -= 2 * eps
            lm = loss(q)
            fd[idx] = (lp - lm) / (2 * eps)
        err = relerr(b[grad_name], fd)
        assert err <= 1e-6, (name, err)


# ----------------------------------------------------------------------------
# forward: library MLP special cases


def test_alpha_zero_is_library_swiglu_mlp():
    rng = np.random.default_rng(1)
    p, _ = rand_params(rng, 9, 12, 20, 4)
    out = oracle.forward(p, 0.0)["out"]
    t = {k: torch.from_numpy(v) for k, v in p.items()}
    ref = library_mlp(t["X"], t["Wg"], t["Wu"], t["Wd"]).numpy()
    assert relerr(out, ref) <= 1e-12


def test_merged_weight_equivalence_forward_and_backward():
    """W' = W + s B A applied densely gives the same out and dX; the dense
    weight gradient maps to the adapter gradients by dA = s B^T dW', dB = s dW' A^T.
    The dense side is torch autograd (float64), a separate implementation."""
    rng = np.random.default_rng(2)
    N, d, d_ff, r, alpha = 11, 13, 17, 5, 7.0
    s = alpha / r
    p, dOut = rand_params(rng, N, d, d_ff, r)
    f = oracle.forward(p, alpha)
    b = oracle.backward(p, alpha, dOut, f)

    t = {k: torch.from_numpy(v.copy()) for k, v in p.items()}
    Wg_m = (t["Wg"] + s * t["Bg"] @ t["Ag"]).requires_grad_(True)
    Wu_m = (t["Wu"] + s * t["Bu"] @ t["Au"]).requires_grad_(True)
    Wd_m = (t["Wd"] + s * t["Bd"] @ t["Ad"]).requires_grad_(True)
    X = t["X"].clone().requires_grad_(True)
    out = library_mlp(X, Wg_m, Wu_m, Wd_m)
    out.backward(torch.from_numpy(dOut))
    assert relerr(f["out"], out.detach().numpy()) <= 1e-12
    assert relerr(b["dX"], X.grad.numpy()) <= 1e-12
    for W, A, B, dA, dB in ((Wg_m, "Ag", "Bg", "dAg", "dBg"),
                             (Wu_m, "Au", "Bu", "dAu", "dBu"),
                             (Wd_m, "Ad", "Bd", "dAd", "dBd")):
        dW = W.grad.numpy()
        assert relerr(b[dA], s * p[B].T @ dW) <= 1e-12, dA
        assert relerr(b[dB], s * dW @ p[A].T) <= 1e-12, dB


def test_zero_B_gives_frozen_mlp_exactly():
    rng = np.random.default_rng(3)
    p, dOut = rand_params(rng, 6, 8, 12, 3)
    pz = dict(p)
    for k in ("Bg", "Bu", "Bd"):
        pz[k] = np.zeros_like(p[k])
    out_z = oracle.forward(pz, 5.0)["out"]
    out_frozen = oracle.forward(p, 0.0)["out"]
    assert np.array_equal(out_z, out_frozen)
    b = oracle.backward(pz, 5.0, dOut)
    for k in ("dAg", "dAu", "dAd"):
        assert np.all(b[k] == 0.0), k
    for k in ("dBg", "dBu", "dBd"):
        assert np.max(np.abs(b[k])) > 0, k


@pytest.mark.parametrize("c", [3.0, -0.25])
def test_adapter_rescaling_invariance(c):
    """(A, B) -> (c A, B / c) leaves out and dX unchanged, dA -> dA / c, dB -> c dB."""
    rng = np.random.default_rng(4)
    alpha = 2.0
    p, dOut = rand_params(rng, 7, 9, 14, 3)
    q = dict(p)
    for a, bb in (("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd")):
        q[a] = c * p[a]
        q[bb] = p[bb] / c
    f0, f1 = oracle.forward(p, alpha), oracle.forward(q, alpha)
    b0, b1 = oracle.backward(p, alpha, dOut, f0), oracle.backward(q, alpha, dOut, f1)
    assert relerr(f1["out"], f0["out"]) <= 1e-12
    assert relerr(b1["dX"], b0["dX"]) <= 1e-12
    for a, bb in (("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd")):
        assert relerr(b1["d" + a], b0["d" + a] / c) <= 1e-12
        assert relerr(b1["d" + bb], b0["d" + bb] * c) <= 1e-12


def test_general_invertible_reparameterisation():
    """A -> M A, B -> B M^-1 for an invertible r x r M leaves out unchanged."""
    rng = np.random.default_rng(5)
    p, _ = rand_params(rng, 5, 8, 10, 4)
    M = rng.standard_normal((4, 4)) + 4 * np.eye(4)
    Mi = np.linalg.inv(M)
    q = dict(p)
    for a, bb in (("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd")):
        q[a] = M @ p[a]
        q[bb] = p[bb] @ Mi
    assert relerr(oracle.forward(q, 3.0)["out"], oracle.forward(p, 3.0)["out"]) <= 1e-11


def test_zero_input_gives_zero_everything():
    rng = np.random.default_rng(6)
    p, dOut = rand_params(rng, 4, 6, 8, 2)
    p["X"] = np.zeros_like(p["X"])
    f = oracle.forward(p, 2.0)
    b = oracle.backward(p, 2.0, dOut, f)
    assert np.all(f["out"] == 0)
    for k in ("dX", "dAg", "dBg", "dAu", "dBu", "dAd", "dBd"):
        assert np.all(b[k] == 0), k


def test_gate_at_zero_halves_the_up_path():
    """At G = 0, sigmoid = 1/2 and dG = dH * U / 2."""
    rng = np.random.default_rng(8)
    p, dOut = rand_params(rng, 3, 4, 5, 2)
    p["Wg"] = np.zeros_like(p["Wg"])
    p["Bg"] = np.zeros_like(p["Bg"])
    f = oracle.forward(p, 1.0)
    b = oracle.backward(p, 1.0, dOut, f)
    assert np.all(f["G"] == 0)
    assert np.allclose(b["dG"], b["dH"] * f["U"] / 2, rtol=0, atol=1e-15)


def test_scalar_closed_form(golden_dir):
    with open(os.path.join(golden_dir, "scalar_closed_form.json")) as fh:
        g = json.load(fh)
    L = math.log(3.0)
    env = {"L": L}
    p = {}
    for k, v in g["inputs"].items():
        p[k] = np.array(eval(v, {}, env) if isinstance(v, str) else v, dtype=np.float64)
    dOut = p.pop("dOut")
    f = oracle.forward(p, g["alpha"])
    b = oracle.backward(p, g["alpha"], dOut, f)
    both = dict(f)
    both.update(b)
    for k, expr in g["expected"].items():
        want = eval(expr, {}, env)
        assert abs(float(both[k].ravel()[0]) - want) <= 1e-14 * max(1.0, abs(want)), k


# ----------------------------------------------------------------------------
# int4 dequantisation


def _round_fraction_rne(x: Fraction, mant_bits: int) -> Fraction:
    """Round a non-zero rational to the nearest binary float with `mant_bits`
    explicit significand bits (normal range), ties to even."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - mant_bits)
    m = a / ulp
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * lo * ulp


def _bf16_bits_of(v: Fraction) -> int:
    f = float(v)  # exactly representable (8 significand bits)
    return int(np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16)


def test_dequant_matches_exact_rational_double_rounding():
    rng = np.random.default_rng(9)
    scales = list(rng.uniform(1e-3, 4.0, 40).astype(np.float16))
    scales += [np.float16(6e-8), np.float16(1e-5), np.float16(65504.0), np.float16(0.0), np.float16(1.0)]
    codes = np.arange(-8, 8)
    rows = len(scales)
    q = np.tile(codes, (rows, 4))                       # [rows, 64]
    nib = (q & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    sc = np.array(scales, dtype=np.float16).reshape(rows, 1)
    got = oracle.dequant_int4(packed, sc)
    for i in range(rows):
        s = Fraction(float(sc[i, 0]))
        for j in range(64):
            exact = Fraction(int(q[i, j])) * s / 7
            w32 = _round_fraction_rne(exact, 23)
            w16 = _round_fraction_rne(w32, 7)
            want = _bf16_bits_of(w16)
            if exact == 0 and int(q[i, j]) < 0:
                want = 0x8000  # IEEE: a negative code times a +0 scale is -0
            assert int(got[i, j]) == want, (i, j, float(sc[i, 0]), int(q[i, j]))


def test_dequant_nibble_order(golden_dir):
    with open(os.path.join(golden_dir, "int4_nibbles.json")) as fh:
        g = json.load(fh)
    packed = np.zeros((1, 32), dtype=np.uint8)
    for k, b in enumerate(g["bytes_head"]):
        packed[0, k] = int(b, 16)
    sc = np.array([[g["scale"]]], dtype=np.float16)
    vals = oracle.bf16_to_f64(oracle.dequant_int4(packed, sc))[0]
    n = len(g["codes_head"])
    assert list(vals[:n]) == [float(c) for c in g["codes_head"]]
    assert np.all(vals[n:] == 0)


def test_quantiser_round_trip_bound():
    rng = np.random.default_rng(10)
    w = rng.standard_normal((8, 256)).astype(np.float32)
    w[3, 64:128] = 0.0
    packed, sc = synth.quantize_int4(w)
    back = oracle.bf16_to_f64(oracle.dequant_int4(packed, sc))
    blocks = np.abs(w).reshape(8, 4, 64).max(axis=2)
    tol = np.repeat(blocks, 64, axis=1) * (1 / 14 + 2e-3) + 1e-6
    assert np.all(np.abs(back - w) <= tol)
    assert np.all(back[3, 64:128] == 0)


def test_bf16_widen_and_round():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x4049, 0x7F7F], dtype=np.uint16)
    assert list(oracle.bf16_to_f64(bits)) == [1.0, -1.0, 0.0, 3.140625, float(np.float32(3.3895314e38))]
    # ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> 1
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], dtype=np.float32)
    assert list(oracle.f32_to_bf16_rne(x)) == [0x3F80, 0x3F82, 0xBF80]


# ----------------------------------------------------------------------------
# sampled evaluators agree with the full evaluation


def test_sampled_rows_and_features_agree_with_full():
    cfg = synth.custom(40, 64, 96, 8, 16.0, seed_index=11)
    inp = synth.make_inputs(cfg)
    full = oracle.forward_backward(inp, cfg.alpha)
    rows = [0, 7, 39]
    tr = oracle.token_rows(inp, cfg.alpha, rows)
    for k, kk in (("out", "out"), ("G", "G"), ("U", "U"), ("dX", "dX")):
        assert relerr(tr[k], full[kk][rows]) <= 1e-13, k
    feats = [0, 50, 95]
    fg = oracle.up_gate_feature_grads(inp, cfg.alpha, feats)
    assert relerr(fg["dBg"], full["dBg"][feats]) <= 1e-13
    assert relerr(fg["dBu"], full["dBu"][feats]) <= 1e-13


def test_int4_inputs_route_through_dequant():
    cfg = synth.custom(16, 64, 128, 8, 8.0, int4=True, seed_index=12)
    inp = synth.make_inputs(cfg)
    assert "Wg" not in inp and "Wg_q" in inp
    p = oracle.weights_f64(inp)
    assert np.array_equal(p["Wd"], oracle.bf16_to_f64(oracle.dequant_int4(inp["Wd_q"], inp["Wd_scale"])))
