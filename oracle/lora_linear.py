"""fp64 CPU oracle of a LoRA-adapted linear layer (forward and backward).

TEST INFRASTRUCTURE ONLY (tests/, bench.py's CPU legs); shares no code with
the CUDA path.

What it follows: "Unsloth 还是 AirLLM？一个炼丹，一个硬跑" (blog.cn-res.vip),
section 核心原理（为什么它快）— matrix multiplies and LoRA fused into single
kernels, the fusion the LoRA MLP applies to each of its projections; applied
here to one projection on its own (the attention q/k/v/o case).  The pages
print no formula; this is the plain definition with s = alpha / r in the
nn.Linear layout (W [out, in], A [r, in], B [out, r]):
    Y = X (W + s B A)^T = X W^T + s (X A^T) B^T
and its chain rule for an upstream gradient dY (W frozen):
    T = s dY B,  dX = dY W + T A,  dA = T^T X,  dB = s dY^T (X A^T).
float64 throughout, numpy matmul as the only library step.
"""
from __future__ import annotations

import numpy as np

from .lora_mlp import bf16_to_f64, dequant_fp8, dequant_int4


def forward(p: dict, alpha: float) -> dict:
    r = p["A"].shape[0]
    s = alpha / r
    R = p["X"] @ p["A"].T                      # [N, r]
    Y = p["X"] @ p["W"].T + s * (R @ p["B"].T)  # [N, out]
    return {"s": s, "R": R, "Y": Y}


def backward(p: dict, alpha: float, dY: np.ndarray, fwd: dict | None = None) -> dict:
    f = forward(p, alpha) if fwd is None else fwd
    s = f["s"]
    T = s * (dY @ p["B"])                       # [N, r]
    dX = dY @ p["W"] + T @ p["A"]               # [N, in]
    dA = T.T @ p["X"]                           # [r, in]
    dB = s * (dY.T @ f["R"])                    # [out, r]
    return {"dX": dX, "dA": dA, "dB": dB, "T": T}


def weights_f64(inputs: dict) -> dict:
    p = {k: bf16_to_f64(v) for k, v in inputs.items() if k in ("X", "W", "A", "B", "dY")}
    if "W" not in p and "W_q" in inputs:
        p["W"] = bf16_to_f64(dequant_int4(inputs["W_q"], inputs["W_scale"]))
    elif "W" not in p:
        p["W"] = bf16_to_f64(dequant_fp8(inputs["W_f8"], inputs["W_f8scale"]))
    return p


def forward_backward(inputs: dict, alpha: float) -> dict:
    p = weights_f64(inputs)
    f = forward(p, alpha)
    b = backward(p, alpha, p["dY"], f)
    res = dict(f)
    res.update(b)
    return res
