"""fp64 CPU oracle of the fused LoRA + SwiGLU MLP (forward, hand-derived backward,
dequantisation of block-int4 and block-FP8 frozen weights).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only tests/, __graft_entry__.smoke() and bench.py (its CPU-baseline leg and
its `--impl reference` arm) may call it.  It shares no code with the CUDA path.

What it follows.
  * "Unsloth 深度分析报告" (nightvoyager.top), section 核心价值提炼 / 创新之处,
    item "融合 LoRA MLP 反向传播 Kernel": the gate, up and down projections of a
    SwiGLU MLP each carry a LoRA adapter; forward and backward of all three are
    fused into one autograd function whose gradients are derived by hand, so
    the intermediates autograd would keep are never stored.
  * Same report, section 关键设计决策: SwiGLU and the LoRA MLP are among the
    six hand-written kernel families.
  * "Unsloth 还是 AirLLM？一个炼丹，一个硬跑" (blog.cn-res.vip), section
    核心原理（为什么它快） / "Why it is fast": matrix multiplies and LoRA fused
    into single kernels; native 4-bit QLoRA for the frozen weights; FP8 and
    NVFP4 named as weight formats.
  * "Unsloth 深度分析报告", section 关键设计决策: FP8 among the hand-written
    kernel families.
The pages print no formula.  The forward used here is the plain definition of
a LoRA-adapted SwiGLU MLP with scale s = alpha / r,
    G = X (Wg + s Bg Ag)^T,  U = X (Wu + s Bu Au)^T,  H = silu(G) * U,
    out = H (Wd + s Bd Ad)^T,
in the nn.Linear layout (W [out, in], A [r, in], B [out, r]).  The backward
is that forward's chain rule, written out below; the int4 format is symmetric
codes in [-7, 7], one fp16 absmax scale per 64 input elements, w = q*scale/7;
the FP8 format is E4M3 codes with one fp32 scale per 64 input elements,
w = e4m3 * scale.

Everything is evaluated in float64 from the exact values of the bf16 inputs,
with every intermediate materialised.  numpy's matmul is the only library
step.  Nothing is blocked, fused or reordered.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# storage formats


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of a bf16 bit pattern (uint16) as float64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def dequant_int4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantise a block-int4 weight to bf16 bits.

    packed: uint8 [rows, cols/2], element 2k in the low nibble of byte k,
    two's-complement nibbles.  scales: float16 [rows, cols/64].
    Per element, in IEEE fp32: w = (fp32(q) * fp32(scale)) / 7, then rounded
    to bf16 (nearest, ties to even).  The product is exact in fp32
    (|q| <= 8 times an 11-bit significand); the division is correctly rounded.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    cols = 2 * half
    codes = np.empty((rows, cols), dtype=np.int16)
    codes[:, 0::2] = packed & 0x0F
    codes[:, 1::2] = packed >> 4
    codes = np.where(codes >= 8, codes - 16, codes)
    scale32 = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float32), 64, axis=1)
    assert scale32.shape == (rows, cols)
    prod = codes.astype(np.float32) * scale32          # exact in fp32
    w32 = prod / np.float32(7.0)                       # IEEE fp32 divide
    return f32_to_bf16_rne(w32)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact values of FP8 E4M3 codes (the OCP 8-bit floating point format
    "E4M3": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; an
    exponent field of 0 encodes subnormals, m/8 * 2^-6; no infinities; the
    two codes S.1111.111 are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequant_fp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantise a block-FP8 weight to bf16 bits.

    codes: uint8 [rows, cols], FP8 E4M3 (see e4m3_to_f64).  scales: float32
    [rows, cols/64], one per 64 consecutive input-dimension elements.
    Per element, in IEEE fp32: w = fp32(e4m3) * scale (one rounding), then
    rounded to bf16 (nearest, ties to even).  fp32(e4m3) is exact (3
    mantissa bits, exponents -9..8).
    """
    codes = np.asarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    v32 = e4m3_to_f64(codes).astype(np.float32)          # exact
    s32 = np.repeat(np.asarray(scales, dtype=np.float32), 64, axis=1)
    assert s32.shape == (rows, cols)
    with np.errstate(invalid="ignore", over="ignore"):
        w32 = v32 * s32                                   # IEEE fp32 multiply
    return f32_to_bf16_rne(w32)


def weights_f64(inputs: dict) -> dict:
    """All float inputs widened to float64; quantised frozen weights
    (int4: '<W>_q', '<W>_scale'; FP8: '<W>_f8', '<W>_f8scale') dequantised first."""
    p = {}
    for k, v in inputs.items():
        if k.endswith(("_q", "_scale", "_f8", "_f8scale")):
            continue
        p[k] = bf16_to_f64(v)
    for w in ("Wg", "Wu", "Wd"):
        if w not in p and w + "_q" in inputs:
            p[w] = bf16_to_f64(dequant_int4(inputs[w + "_q"], inputs[w + "_scale"]))
        elif w not in p and w + "_f8" in inputs:
            p[w] = bf16_to_f64(dequant_fp8(inputs[w + "_f8"], inputs[w + "_f8scale"]))
    return p


# ----------------------------------------------------------------------------
# the MLP


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def forward(p: dict, alpha: float, r: int | None = None) -> dict:
    """Forward pass.  p holds float64 X, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd."""
    r = p["Ag"].shape[0] if r is None else r
    s = alpha / r
    X = p["X"]
    R_g = X @ p["Ag"].T                                  # [N, r]
    R_u = X @ p["Au"].T                                  # [N, r]
    G = X @ p["Wg"].T + s * (R_g @ p["Bg"].T)            # [N, d_ff]
    U = X @ p["Wu"].T + s * (R_u @ p["Bu"].T)            # [N, d_ff]
    sig = sigmoid(G)
    silu = G * sig
    H = silu * U
    Q_d = H @ p["Ad"].T                                  # [N, r]
    out = H @ p["Wd"].T + s * (Q_d @ p["Bd"].T)          # [N, d]
    return {"s": s, "R_g": R_g, "R_u": R_u, "G": G, "U": U, "sig": sig,
            "silu": silu, "H": H, "Q_d": Q_d, "out": out}


def backward(p: dict, alpha: float, dOut: np.ndarray, fwd: dict | None = None) -> dict:
    """Chain rule of forward() for the upstream gradient dOut [N, d].

    Returns dX and the gradients of the six adapter matrices (the frozen W get
    none).  With T_d = s dOut Bd, T_g = s dG Bg, T_u = s dU Bu:
      dH  = dOut Wd + T_d Ad
      dBd = s dOut^T Q_d,     dAd = T_d^T H
      dU  = dH * silu(G)
      dG  = dH * U * sig(G) * (1 + G (1 - sig(G)))
      dX  = dG Wg + T_g Ag + dU Wu + T_u Au
      dBg = s dG^T R_g,  dAg = T_g^T X   (and likewise for the up adapter)
    """
    f = forward(p, alpha) if fwd is None else fwd
    s = f["s"]
    X = p["X"]
    T_d = s * (dOut @ p["Bd"])                           # [N, r]
    dH = dOut @ p["Wd"] + T_d @ p["Ad"]                  # [N, d_ff]
    dBd = s * (dOut.T @ f["Q_d"])                        # [d, r]
    dAd = T_d.T @ f["H"]                                 # [r, d_ff]
    dU = dH * f["silu"]
    dG = dH * f["U"] * f["sig"] * (1.0 + f["G"] * (1.0 - f["sig"]))
    T_g = s * (dG @ p["Bg"])                             # [N, r]
    T_u = s * (dU @ p["Bu"])                             # [N, r]
    dX = dG @ p["Wg"] + T_g @ p["Ag"] + dU @ p["Wu"] + T_u @ p["Au"]
    dBg = s * (dG.T @ f["R_g"])                          # [d_ff, r]
    dAg = T_g.T @ X                                      # [r, d]
    dBu = s * (dU.T @ f["R_u"])
    dAu = T_u.T @ X
    return {"dX": dX, "dAg": dAg, "dBg": dBg, "dAu": dAu, "dBu": dBu,
            "dAd": dAd, "dBd": dBd, "dG": dG, "dU": dU, "dH": dH}


def forward_backward(inputs: dict, alpha: float) -> dict:
    """Full forward + backward from the bf16 input dict (see inputs.make_inputs)."""
    p = weights_f64(inputs)
    f = forward(p, alpha)
    b = backward(p, alpha, p["dOut"], f)
    res = dict(f)
    res.update(b)
    return res


# ----------------------------------------------------------------------------
# sampled evaluation for large workloads (each output computed one by one)


def token_rows(inputs: dict, alpha: float, rows) -> dict:
    """out, G, U and dX for a subset of tokens.

    Every token is independent in the MLP, so these rows are forward/backward on
    the sub-batch X[rows], dOut[rows].  (Adapter gradients of a sub-batch are
    partial sums and are not returned.)
    """
    rows = np.asarray(rows)
    sub = {}
    for k, v in inputs.items():
        sub[k] = v[rows] if k in ("X", "dOut") else v
    p = weights_f64(sub)
    f = forward(p, alpha)
    b = backward(p, alpha, p["dOut"], f)
    return {"out": f["out"], "G": f["G"], "U": f["U"], "dX": b["dX"]}


def up_gate_feature_grads(inputs: dict, alpha: float, feats) -> dict:
    """Rows dBg[f, :], dBu[f, :] for a subset of hidden features f.

    Column f of G, U and dH only needs column f of the projections, so each
    sampled row is exact without the full [N, d_ff] intermediates.
    """
    feats = np.asarray(feats)
    p = weights_f64(inputs)
    r = p["Ag"].shape[0]
    s = alpha / r
    X, dOut = p["X"], p["dOut"]
    R_g = X @ p["Ag"].T
    R_u = X @ p["Au"].T
    G = X @ p["Wg"][feats].T + s * (R_g @ p["Bg"][feats].T)      # [N, |f|]
    U = X @ p["Wu"][feats].T + s * (R_u @ p["Bu"][feats].T)
    T_d = s * (dOut @ p["Bd"])
    dH = dOut @ p["Wd"][:, feats] + T_d @ p["Ad"][:, feats]
    sig = sigmoid(G)
    dU = dH * G * sig
    dG = dH * U * sig * (1.0 + G * (1.0 - sig))
    return {"dBg": s * (dG.T @ R_g), "dBu": s * (dU.T @ R_u)}
