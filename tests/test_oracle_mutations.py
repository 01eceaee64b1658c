"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's arithmetic (a dropped
term, a wrong sign, a swapped adapter, a transposed operand, a wrong scale)
on the CPU and checks that the finite-difference or library-MLP pins reject
it, while the unmodified oracle passes the same checks."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import lora_mlp as om


def params(seed=3, N=4, d=6, d_ff=9, r=3):
    rng = np.random.default_rng(seed)
    p = {
        "X": rng.standard_normal((N, d)),
        "Wg": rng.standard_normal((d_ff, d)) / math.sqrt(d),
        "Wu": rng.standard_normal((d_ff, d)) / math.sqrt(d),
        "Wd": rng.standard_normal((d, d_ff)) / math.sqrt(d_ff),
        "Ag": rng.uniform(-1, 1, (r, d)),
        "Bg": rng.standard_normal((d_ff, r)) * 0.3,
        "Au": rng.uniform(-1, 1, (r, d)),
        "Bu": rng.standard_normal((d_ff, r)) * 0.3,
        "Ad": rng.uniform(-1, 1, (r, d_ff)),
        "Bd": rng.standard_normal((d, r)) * 0.3,
    }
    return p, rng.standard_normal((N, d))


def fd_pin_holds(fwd, bwd, alpha=2.5):
    """Central differences of <dOut, out> agree with the analytic gradients."""
    p, dOut = params()
    b = bwd(p, alpha, dOut)
    for name, g in [("X", "dX"), ("Ag", "dAg"), ("Bg", "dBg"), ("Au", "dAu"), ("Bu", "dBu"), ("Ad", "dAd"),
                    ("Bd", "dBd")]:
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(*p[name].shape):
            q = {k: v.copy() for k, v in p.items()}
            q[name][idx] += 1e-5
            lp = float(np.sum(dOut * fwd(q, alpha)["out"]))
            q[name][idx] -= 2e-5
            lm = float(np.sum(dOut * fwd(q, alpha)["out"]))
            fd[idx] = (lp - lm) / 2e-5
        if np.max(np.abs(fd - b[g])) > 1e-6 * max(np.max(np.abs(b[g])), 1e-30):
            return False
    return True


def merged_pin_holds(fwd, alpha=2.5):
    """out equals a library SwiGLU MLP on the merged weights W + s B A."""
    p, _ = params()
    s = alpha / p["Ag"].shape[0]
    t = {k: torch.from_numpy(v) for k, v in p.items()}
    F = torch.nn.functional
    Wg = t["Wg"] + s * t["Bg"] @ t["Ag"]
    Wu = t["Wu"] + s * t["Bu"] @ t["Au"]
    Wd = t["Wd"] + s * t["Bd"] @ t["Ad"]
    ref = ((F.silu(t["X"] @ Wg.T) * (t["X"] @ Wu.T)) @ Wd.T).numpy()
    out = fwd(p, alpha)["out"]
    return np.max(np.abs(out - ref)) <= 1e-12 * np.max(np.abs(ref))


def mutated_forward(kind):
    def fwd(p, alpha, r=None):
        q = dict(p)
        r_ = p["Ag"].shape[0]
        s = alpha / r_
        if kind == "swap_adapters":
            q["Bg"], q["Bu"] = p["Bu"], p["Bg"]
        if kind == "scale_alpha_only":
            s = alpha
        X = q["X"]
        R_g = X @ q["Ag"].T
        R_u = X @ q["Au"].T
        G = X @ q["Wg"].T + s * (R_g @ q["Bg"].T)
        U = X @ q["Wu"].T + s * (R_u @ q["Bu"].T)
        sig = om.sigmoid(G)
        silu = G * sig if kind != "silu_is_sigmoid" else sig
        H = silu * U
        Q_d = H @ q["Ad"].T
        out = H @ q["Wd"].T + s * (Q_d @ q["Bd"].T)
        return {"s": s, "R_g": R_g, "R_u": R_u, "G": G, "U": U, "sig": sig, "silu": silu, "H": H, "Q_d": Q_d,
                "out": out}
    return fwd


def mutated_backward(kind):
    def bwd(p, alpha, dOut, fwd=None):
        f = om.forward(p, alpha)
        s = f["s"]
        X = p["X"]
        T_d = s * (dOut @ p["Bd"])
        dH = dOut @ p["Wd"] + T_d @ p["Ad"]
        dBd = s * (dOut.T @ f["Q_d"])
        dAd = T_d.T @ f["H"]
        dU = dH * f["silu"]
        if kind == "drop_curvature_term":
            dG = dH * f["U"] * f["sig"]
        elif kind == "wrong_sign":
            dG = dH * f["U"] * f["sig"] * (1.0 - f["G"] * (1.0 - f["sig"]))
        else:
            dG = dH * f["U"] * f["sig"] * (1.0 + f["G"] * (1.0 - f["sig"]))
        T_g = s * (dG @ p["Bg"])
        T_u = s * (dU @ p["Bu"])
        if kind == "missing_lora_dx":
            dX = dG @ p["Wg"] + dU @ p["Wu"]
        else:
            dX = dG @ p["Wg"] + T_g @ p["Ag"] + dU @ p["Wu"] + T_u @ p["Au"]
        dBg = s * (dG.T @ f["R_g"])
        dAg = T_g.T @ X
        if kind == "transposed_dB_operand":
            dBg = s * (dG.T @ (X @ p["Au"].T))
        dBu = s * (dU.T @ f["R_u"])
        dAu = T_u.T @ X
        return {"dX": dX, "dAg": dAg, "dBg": dBg, "dAu": dAu, "dBu": dBu, "dAd": dAd, "dBd": dBd}
    return bwd


def test_unmodified_oracle_passes_both_pins():
    assert fd_pin_holds(oracle.forward, oracle.backward)
    assert merged_pin_holds(oracle.forward)


@pytest.mark.parametrize("kind", ["swap_adapters", "scale_alpha_only", "silu_is_sigmoid"])
def test_forward_mistakes_are_caught(kind):
    assert not merged_pin_holds(mutated_forward(kind))


@pytest.mark.parametrize("kind", ["drop_curvature_term", "wrong_sign", "missing_lora_dx", "transposed_dB_operand"])
def test_backward_mistakes_are_caught(kind):
    assert not fd_pin_holds(oracle.forward, mutated_backward(kind))


# ----------------------------------------------------------------------------- RMSNorm

from oracle import rmsnorm as orn  # noqa: E402


def rms_pins_hold(fwd, bwd):
    """Library rms_norm (forward + autograd backward) and central differences."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((5, 12)) * rng.uniform(0.2, 4.0, (5, 1))
    gamma = rng.uniform(0.5, 1.5, 12)
    dy = rng.standard_normal((5, 12))
    eps = 1e-3
    y, rstd = fwd(x, gamma, eps)
    tx = torch.from_numpy(x.copy()).requires_grad_(True)
    ty = torch.nn.functional.rms_norm(tx, (12,), torch.from_numpy(gamma), eps=eps)
    ty.backward(torch.from_numpy(dy))
    if np.max(np.abs(y - ty.detach().numpy())) > 1e-12:
        return False
    dx = bwd(x, gamma, rstd, dy)
    return bool(np.max(np.abs(dx - tx.grad.numpy())) <= 1e-10 * np.max(np.abs(dx)))


def test_rmsnorm_pins_accept_the_oracle():
    assert rms_pins_hold(orn.rmsnorm_forward, orn.rmsnorm_backward)


RMS_MUTANTS = {
    # variance about the mean instead of the mean square
    "centred": (lambda x, g, e: (x * (1 / np.sqrt(np.var(x, axis=1) + e))[:, None] * g,
                                 1 / np.sqrt(np.var(x, axis=1) + e)), orn.rmsnorm_backward),
    # eps outside the square root
    "eps_outside": (lambda x, g, e: (x * (1 / (np.sqrt(np.mean(x * x, axis=1)) + e))[:, None] * g,
                                     1 / (np.sqrt(np.mean(x * x, axis=1)) + e)), orn.rmsnorm_backward),
    # backward drops the projection term
    "no_projection": (orn.rmsnorm_forward, lambda x, g, r, dy: r[:, None] * dy * g),
    # backward forgets gamma inside the projection
    "gamma_outside_mean": (orn.rmsnorm_forward,
                           lambda x, g, r, dy: r[:, None] * (dy * g - (x * r[:, None]) * np.mean(
                               dy * x * r[:, None], axis=1)[:, None])),
    # backward uses sum instead of mean
    "sum_not_mean": (orn.rmsnorm_forward,
                     lambda x, g, r, dy: r[:, None] * (dy * g - (x * r[:, None]) * np.sum(
                         dy * g * x * r[:, None], axis=1)[:, None])),
}


@pytest.mark.parametrize("name", sorted(RMS_MUTANTS))
def test_rmsnorm_pins_reject_mutant(name):
    fwd, bwd = RMS_MUTANTS[name]
    assert not rms_pins_hold(fwd, bwd)
