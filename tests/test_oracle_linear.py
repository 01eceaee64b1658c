"""Pins for the LoRA linear oracle: central finite differences, a library
linear layer with merged weights under torch autograd, B = 0 and adapter
rescaling."""
import math

import numpy as np
import pytest
import torch

from oracle import lora_linear as ol


def params(seed, N, di, do, r):
    rng = np.random.default_rng(seed)
    p = {"X": rng.standard_normal((N, di)), "W": rng.standard_normal((do, di)) / math.sqrt(di),
         "A": rng.uniform(-1, 1, (r, di)), "B": rng.standard_normal((do, r)) * 0.3}
    return p, rng.standard_normal((N, do))


def relerr(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("shape", [(3, 5, 7, 2), (4, 6, 3, 3)])
def test_backward_matches_central_differences(shape):
    p, dY = params(1, *shape)
    alpha = 2.5
    b = ol.backward(p, alpha, dY)
    for name, g in (("X", "dX"), ("A", "dA"), ("B", "dB")):
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(*p[name].shape):
            q = {k: v.copy() for k, v in p.items()}
            q[name][idx] += 1e-5
            lp = float(np.sum(dY * ol.forward(q, alpha)["Y"]))
            q[name][idx] -= 2e-5
            lm = float(np.sum(dY * ol.forward(q, alpha)["Y"]))
            fd[idx] = (lp - lm) / 2e-5
        assert relerr(b[g], fd) <= 1e-6, name


def test_merged_weight_library_linear_with_autograd():
    p, dY = params(2, 9, 11, 13, 4)
    alpha = 6.0
    s = alpha / 4
    f = ol.forward(p, alpha)
    b = ol.backward(p, alpha, dY, f)
    t = {k: torch.from_numpy(v.copy()) for k, v in p.items()}
    Wm = (t["W"] + s * t["B"] @ t["A"]).requires_grad_(True)
    X = t["X"].clone().requires_grad_(True)
    Y = torch.nn.functional.linear(X, Wm)
    Y.backward(torch.from_numpy(dY))
    assert relerr(f["Y"], Y.detach().numpy()) <= 1e-12
    assert relerr(b["dX"], X.grad.numpy()) <= 1e-12
    dW = Wm.grad.numpy()
    assert relerr(b["dA"], s * p["B"].T @ dW) <= 1e-12
    assert relerr(b["dB"], s * dW @ p["A"].T) <= 1e-12


def test_zero_B_and_rescaling():
    p, dY = params(3, 5, 6, 7, 3)
    q = dict(p)
    q["B"] = np.zeros_like(p["B"])
    assert np.array_equal(ol.forward(q, 3.0)["Y"], ol.forward(p, 0.0)["Y"])
    assert np.all(ol.backward(q, 3.0, dY)["dA"] == 0)
    c = 2.0
    q = dict(p)
    q["A"], q["B"] = c * p["A"], p["B"] / c
    b0, b1 = ol.backward(p, 3.0, dY), ol.backward(q, 3.0, dY)
    assert relerr(b1["dX"], b0["dX"]) <= 1e-12
    assert relerr(b1["dA"], b0["dA"] / c) <= 1e-12
    assert relerr(b1["dB"], b0["dB"] * c) <= 1e-12
