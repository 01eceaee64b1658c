"""Pins for the RMSNorm / pre-norm block oracle: torch's library rms_norm
(forward and autograd backward) in float64, central finite differences of
the whole block, and the closed-form invariants of RMS normalisation."""
import math

import numpy as np
import pytest
import torch

from oracle import lora_mlp as om
from oracle import rmsnorm as orn
from lora_fine_tuning_mlp_b200 import inputs as synth


def relerr(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("eps", [0.0, 1e-5, 0.3])
def test_forward_and_backward_match_torch_rms_norm(eps):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 24)) * rng.uniform(0.1, 5.0, (7, 1))
    gamma = rng.uniform(0.5, 1.5, 24)
    dy = rng.standard_normal((7, 24))
    y, rstd = orn.rmsnorm_forward(x, gamma, eps)
    dx = orn.rmsnorm_backward(x, gamma, rstd, dy)
    tx = torch.from_numpy(x.copy()).requires_grad_(True)
    ty = torch.nn.functional.rms_norm(tx, (24,), torch.from_numpy(gamma), eps=eps)
    ty.backward(torch.from_numpy(dy))
    assert relerr(y, ty.detach().numpy()) <= 1e-13
    assert relerr(dx, tx.grad.numpy()) <= 1e-12


def test_invariants_at_zero_eps():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 16))
    gamma = rng.uniform(0.5, 1.5, 16)
    dy = rng.standard_normal((5, 16))
    y1, r1 = orn.rmsnorm_forward(x, np.ones(16), 0.0)
    assert np.allclose(np.mean(y1 * y1, axis=1), 1.0, rtol=1e-14)          # unit RMS
    y, rstd = orn.rmsnorm_forward(x, gamma, 0.0)
    y3, r3 = orn.rmsnorm_forward(3.0 * x, gamma, 0.0)
    assert relerr(y3, y) <= 1e-14 and relerr(r3, r1 / 3.0) <= 1e-14         # scale invariance
    dx = orn.rmsnorm_backward(x, gamma, rstd, dy)
    assert np.max(np.abs(np.sum(dx * x, axis=1))) <= 1e-12 * np.max(np.abs(dx))  # no gradient along x
    dx3 = orn.rmsnorm_backward(3.0 * x, gamma, r3, dy)
    assert relerr(dx3, dx / 3.0) <= 1e-13


@pytest.mark.parametrize("shape", [(3, 8, 6, 2), (4, 6, 10, 3)])
def test_block_backward_matches_central_differences(shape):
    N, d, d_ff, r = shape
    rng = np.random.default_rng(7)
    p = {"X": rng.standard_normal((N, d)) * rng.uniform(0.3, 3.0, (N, 1)),
         "Wg": rng.standard_normal((d_ff, d)) / math.sqrt(d), "Wu": rng.standard_normal((d_ff, d)) / math.sqrt(d),
         "Wd": rng.standard_normal((d, d_ff)) / math.sqrt(d_ff),
         "Ag": rng.uniform(-1, 1, (r, d)), "Au": rng.uniform(-1, 1, (r, d)), "Ad": rng.uniform(-1, 1, (r, d_ff)),
         "Bg": rng.standard_normal((d_ff, r)) * 0.3, "Bu": rng.standard_normal((d_ff, r)) * 0.3,
         "Bd": rng.standard_normal((d, r)) * 0.3}
    gamma = rng.uniform(0.5, 1.5, d)
    dOut = rng.standard_normal((N, d))
    alpha, eps = 3.0, 1e-2

    def loss(q):
        xn, _ = orn.rmsnorm_forward(q["X"], gamma, eps)
        qq = dict(q, X=xn)
        return float(np.sum(dOut * om.forward(qq, alpha)["out"]))

    xn, rstd = orn.rmsnorm_forward(p["X"], gamma, eps)
    pn = dict(p, X=xn)
    b = om.backward(pn, alpha, dOut)
    grads = {"X": orn.rmsnorm_backward(p["X"], gamma, rstd, b["dX"]), "Ag": b["dAg"], "Bd": b["dBd"]}
    for name, an in grads.items():
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(*p[name].shape):
            q = {k: v.copy() for k, v in p.items()}
            q[name][idx] += 1e-6
            lp = loss(q)
            q[name][idx] -= 2e-6
            fd[idx] = (lp - loss(q)) / 2e-6
        assert relerr(an, fd) <= 1e-6, name


def test_block_oracle_composes_norm_and_mlp():
    cfg = synth.custom(20, 64, 96, 8, 16.0, seed_index=90)
    inp = synth.make_block_inputs(cfg)
    r = orn.block_forward_backward(inp, cfg.alpha, synth.RMS_EPS)
    gamma = om.bf16_to_f64(inp["gamma"])
    x = om.bf16_to_f64(inp["X"])
    xn = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(gamma), eps=synth.RMS_EPS)
    assert relerr(r["Xn"], xn.numpy()) <= 1e-13
    rows = orn.block_token_rows(inp, cfg.alpha, synth.RMS_EPS, [0, 7, 19])
    for k in ("out", "dX"):
        assert relerr(rows[k], r[k][[0, 7, 19]]) <= 1e-12, k
