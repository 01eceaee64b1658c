"""fp64 CPU oracle of RMSNorm and of the pre-norm LoRA MLP block.

TEST INFRASTRUCTURE ONLY (tests/, bench.py's CPU legs); shares no code with
the CUDA path.

What it follows:
  - "Unsloth 深度分析报告" (nightvoyager.top), section 关键设计决策: an RMS
    layer-norm kernel with forward and backward among the hand-written kernels;
  - "Unsloth支持哪些模型？主流LLM兼容性一览" (pwwt.cn), section 4.2: the
    backward reuses the statistics cached by the forward instead of
    recomputing the mean of squares; section 2.6 quotes rms_norm_eps = 1e-5.
The pages print no formula.  The plain definition, per row x of length d,
with a frozen gain gamma:
    rstd = (mean(x^2) + eps)^(-1/2),   y = x * rstd * gamma
and its chain rule (x_hat = x * rstd, dxh = dy * gamma):
    dx = rstd * (dxh - x_hat * mean(dxh * x_hat)).
The block is out = MLP(RMSNorm(X_res)) with the LoRA SwiGLU MLP of
oracle.lora_mlp; its backward chains the two.  float64 throughout.
"""
from __future__ import annotations

import numpy as np

from . import lora_mlp as om


def rmsnorm_forward(x: np.ndarray, gamma: np.ndarray, eps: float):
    """Returns (y, rstd) for rows of x."""
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=1) + eps)
    return x * rstd[:, None] * gamma[None, :], rstd


def rmsnorm_backward(x: np.ndarray, gamma: np.ndarray, rstd: np.ndarray, dy: np.ndarray) -> np.ndarray:
    """dx for upstream dy, reusing the forward's rstd (no gradient for gamma)."""
    x_hat = x * rstd[:, None]
    dxh = dy * gamma[None, :]
    return rstd[:, None] * (dxh - x_hat * np.mean(dxh * x_hat, axis=1)[:, None])


def block_forward_backward(inputs: dict, alpha: float, eps: float) -> dict:
    """inputs: the MLP inputs of lora_fine_tuning_mlp_b200.inputs with X the
    residual-stream rows (pre-norm) and 'gamma' (bf16 bits, [d])."""
    p = om.weights_f64(inputs)
    gamma = om.bf16_to_f64(inputs["gamma"])
    xr = p["X"]
    xn, rstd = rmsnorm_forward(xr, gamma, eps)
    p["X"] = xn
    f = om.forward(p, alpha)
    b = om.backward(p, alpha, p["dOut"], f)
    res = dict(f)
    res.update(b)
    res["Xn"] = xn
    res["rstd"] = rstd
    res["dXn"] = b["dX"]
    res["dX"] = rmsnorm_backward(xr, gamma, rstd, b["dX"])
    return res


def block_token_rows(inputs: dict, alpha: float, eps: float, rows) -> dict:
    """out, g, u, dX for a subset of tokens (tokens are independent)."""
    rows = np.asarray(rows)
    sub = {k: (v[rows] if k in ("X", "dOut") else v) for k, v in inputs.items()}
    r = block_forward_backward(sub, alpha, eps)
    return {"out": r["out"], "G": r["G"], "U": r["U"], "dX": r["dX"], "rstd": r["rstd"], "Xn": r["Xn"]}
