"""Seeded synthetic inputs for the fused LoRA + SwiGLU MLP.

This module only draws random numbers and rounds them to the storage formats
(bf16, and the int4 and FP8 block formats of the frozen weights).  It holds none of the
arithmetic of the MLP itself, so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any of the method.

Layout (nn.Linear / PEFT convention, row-major):
  X  [N, d]        Wg, Wu [d_ff, d]   Wd [d, d_ff]
  Ag, Au [r, d]    Bg, Bu [d_ff, r]   Ad [r, d_ff]   Bd [d, r]
  dOut [N, d]      (upstream gradient of the MLP output)

Recipe (one numpy PCG64 generator, seed = 1234 + config index, draws in this
order, each drawn in float32 and rounded to bf16 with round-to-nearest-even):
  X ~ N(0, 1); Wg, Wu ~ N(0, 1/d); Wd ~ N(0, 1/d_ff)  (second argument = variance)
  A ~ U(-1/sqrt(fan_in), +1/sqrt(fan_in)), fan_in = d for Ag, Au and d_ff for Ad
  B ~ N(0, 0.02^2)  (std 0.02, non-zero so that every adapter gradient is exercised)
  dOut ~ N(0, 1)

The LoRA linear, pre-norm block and cross-entropy workloads further down
state their own recipes.
"""
from __future__ import annotations

import dataclasses

import numpy as np

NAMES = ("X", "Wg", "Wu", "Wd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd", "dOut")
WEIGHT_NAMES = ("Wg", "Wu", "Wd")
ADAPTER_NAMES = ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")
INT4_BLOCK = 64


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    N: int
    d: int
    d_ff: int
    r: int
    alpha: float
    int4: bool = False
    index: int = 0
    fp8: bool = False

    @property
    def s(self) -> float:
        return self.alpha / self.r

    @property
    def seed(self) -> int:
        return 1234 + self.index

    def flops_fwd(self) -> float:
        """Algorithmic forward flops: three dense projections plus the rank-r paths."""
        return 6.0 * self.N * self.d * self.d_ff + 6.0 * self.N * self.r * (self.d + self.d_ff)

    def flops_bwd(self) -> float:
        """Algorithmic backward flops (no gradient for the frozen dense weights)."""
        return 6.0 * self.N * self.d * self.d_ff + 12.0 * self.N * self.r * (self.d + self.d_ff)

    def flops(self) -> float:
        return self.flops_fwd() + self.flops_bwd()


# The five workloads: a tiny one for full parity, and model-shaped ones.
CONFIGS = (
    Config("tiny", 512, 256, 704, 8, 16.0, index=0),
    Config("tinyllama_mlp", 32768, 2048, 5632, 32, 32.0, index=1),
    Config("llama3_8b_mlp", 4096, 4096, 14336, 16, 16.0, index=2),
    Config("qwen2_7b_mlp", 8192, 3584, 18944, 64, 128.0, index=3),
    Config("llama3_8b_mlp_int4", 4096, 4096, 14336, 16, 16.0, int4=True, index=4),
    Config("llama3_8b_mlp_fp8", 4096, 4096, 14336, 16, 16.0, index=5, fp8=True),
)
BY_NAME = {c.name: c for c in CONFIGS}


def custom(N, d, d_ff, r, alpha, int4=False, seed_index=100, name="custom", fp8=False) -> Config:
    return Config(name, N, d, d_ff, r, float(alpha), int4=int4, index=seed_index, fp8=fp8)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize_int4(w: np.ndarray):
    """Block-quantise a float32 [rows, cols] weight to symmetric int4.

    Blocks of 64 consecutive input-dimension elements share one fp16 scale
    equal to the block's absolute maximum (rounded to fp16).  Codes are
    q = clamp(rint(7 * w / scale), -7, 7); an all-zero block gets scale 0 and
    codes 0.  Packing: element 2k in the low nibble of byte k (two's
    complement), rows packed along the input dimension.
    Returns (packed uint8 [rows, cols/2], scales float16 [rows, cols/64]).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % INT4_BLOCK == 0
    blocks = w.reshape(rows, cols // INT4_BLOCK, INT4_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    scale16 = amax.astype(np.float16)
    scale32 = scale16.astype(np.float32)
    safe = np.where(scale32 > 0, scale32, np.float32(1.0))
    q = np.rint(np.float32(7.0) * blocks / safe[:, :, None])
    q = np.where(scale32[:, :, None] > 0, q, 0.0)
    q = np.clip(q, -7, 7).astype(np.int8).reshape(rows, cols)
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, scale16


FP8_MAX = 448.0  # largest finite E4M3 value


def quantize_fp8(w: np.ndarray):
    """Block-quantise a float32 [rows, cols] weight to FP8 E4M3 codes.

    Blocks of 64 consecutive input-dimension elements share one fp32 scale,
    the block's absolute maximum over 448 (the largest E4M3 value); codes are
    w / scale rounded to E4M3 (nearest, ties to even, by torch's float8_e4m3fn
    conversion).  An all-zero block gets scale 0 and codes 0.
    Returns (codes uint8 [rows, cols], scales float32 [rows, cols/64]).
    """
    import torch

    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % INT4_BLOCK == 0
    blocks = w.reshape(rows, cols // INT4_BLOCK, INT4_BLOCK)
    scale = (np.abs(blocks).max(axis=2) / np.float32(FP8_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0))
    x = np.clip(blocks / safe[:, :, None], -FP8_MAX, FP8_MAX).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(x.reshape(rows, cols))).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8).numpy().copy(), scale


def make_inputs(cfg: Config) -> dict:
    """Draw all inputs of one workload.

    Returns a dict of bf16 bit arrays (uint16) keyed by NAMES.  For int4
    workloads it also holds '<W>_q' (packed uint8) and '<W>_scale' (float16)
    for each frozen weight, for FP8 workloads '<W>_f8' (uint8 E4M3 codes) and
    '<W>_f8scale' (float32); the bf16 '<W>' entry is then absent, because the
    frozen weight only exists in its quantised form.
    """
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    N, d, d_ff, r = cfg.N, cfg.d, cfg.d_ff, cfg.r
    out = {}

    def normal(shape, std):
        return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)

    def uniform(shape, bound):
        return rng.uniform(-bound, bound, size=shape).astype(np.float32)

    f32 = {}
    f32["X"] = normal((N, d), 1.0)
    f32["Wg"] = normal((d_ff, d), 1.0 / np.sqrt(d))
    f32["Wu"] = normal((d_ff, d), 1.0 / np.sqrt(d))
    f32["Wd"] = normal((d, d_ff), 1.0 / np.sqrt(d_ff))
    f32["Ag"] = uniform((r, d), 1.0 / np.sqrt(d))
    f32["Bg"] = normal((d_ff, r), 0.02)
    f32["Au"] = uniform((r, d), 1.0 / np.sqrt(d))
    f32["Bu"] = normal((d_ff, r), 0.02)
    f32["Ad"] = uniform((r, d_ff), 1.0 / np.sqrt(d_ff))
    f32["Bd"] = normal((d, r), 0.02)
    f32["dOut"] = normal((N, d), 1.0)
    for k in NAMES:
        if cfg.int4 and k in WEIGHT_NAMES:
            q, sc = quantize_int4(f32[k])
            out[k + "_q"] = q
            out[k + "_scale"] = sc
        elif cfg.fp8 and k in WEIGHT_NAMES:
            out[k + "_f8"], out[k + "_f8scale"] = quantize_fp8(f32[k])
        else:
            out[k] = f32_to_bf16_bits(f32[k])
        del f32[k]
    return out


def zero_B(inputs: dict) -> dict:
    """Same inputs with every adapter B set to zero (the frozen-MLP special case)."""
    o = dict(inputs)
    for k in ("Bg", "Bu", "Bd"):
        o[k] = np.zeros_like(inputs[k])
    return o


# ----------------------------------------------------------------------------- LoRA linear


@dataclasses.dataclass(frozen=True)
class LinearConfig:
    """One LoRA-adapted projection: X [N, in] -> Y [N, out]."""
    name: str
    N: int
    d_in: int
    d_out: int
    r: int
    alpha: float
    int4: bool = False
    index: int = 50
    fp8: bool = False

    @property
    def seed(self) -> int:
        return 1234 + self.index

    def flops(self) -> float:
        """fwd + bwd: 2 dense products for fwd+dX, rank-r paths, no dW."""
        return 4.0 * self.N * self.d_in * self.d_out + 8.0 * self.N * self.r * (self.d_in + self.d_out)


LINEAR_CONFIGS = (
    LinearConfig("linear_tiny", 300, 192, 320, 8, 16.0, index=50),
    LinearConfig("llama3_8b_qproj", 4096, 4096, 4096, 16, 16.0, index=51),
    LinearConfig("llama3_8b_kproj", 4096, 4096, 1024, 16, 16.0, index=52),
)
LINEAR_BY_NAME = {c.name: c for c in LINEAR_CONFIGS}


def make_linear_inputs(cfg: LinearConfig) -> dict:
    """X ~ N(0,1), W ~ N(0, 1/in), A ~ U(+-1/sqrt(in)), B ~ N(0, 0.02^2),
    dY ~ N(0,1); drawn in this order in fp32 and rounded to bf16 (int4 W:
    the block quantiser above)."""
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    N, di, do, r = cfg.N, cfg.d_in, cfg.d_out, cfg.r
    f32 = {
        "X": rng.standard_normal((N, di), dtype=np.float32),
        "W": rng.standard_normal((do, di), dtype=np.float32) * np.float32(1.0 / np.sqrt(di)),
        "A": rng.uniform(-1.0 / np.sqrt(di), 1.0 / np.sqrt(di), size=(r, di)).astype(np.float32),
        "B": rng.standard_normal((do, r), dtype=np.float32) * np.float32(0.02),
        "dY": rng.standard_normal((N, do), dtype=np.float32),
    }
    out = {}
    for k, v in f32.items():
        if cfg.int4 and k == "W":
            out["W_q"], out["W_scale"] = quantize_int4(v)
        elif cfg.fp8 and k == "W":
            out["W_f8"], out["W_f8scale"] = quantize_fp8(v)
        else:
            out[k] = f32_to_bf16_bits(v)
    return out


# ----------------------------------------------------------------------------- pre-norm block

RMS_EPS = 1e-5


def make_block_inputs(cfg: Config) -> dict:
    """Inputs of the pre-norm block out = MLP(RMSNorm(X)): the MLP inputs of
    `cfg` with every row of X rescaled by a log-uniform factor in [1/4, 4]
    (so rows have different RMS, like a residual stream) and a frozen gain
    gamma ~ U(0.5, 1.5) [d].  Both come from a second generator (seed + 7919),
    so the MLP inputs themselves are unchanged; X is rounded to bf16 again."""
    out = make_inputs(cfg)
    rng = np.random.Generator(np.random.PCG64(cfg.seed + 7919))
    scale = np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=(cfg.N, 1))).astype(np.float32)
    out["X"] = f32_to_bf16_bits(bf16_bits_to_f32(out["X"]) * scale)
    out["gamma"] = f32_to_bf16_bits(rng.uniform(0.5, 1.5, size=cfg.d).astype(np.float32))
    return out


# The block workloads: a name for the pre-norm block on an MLP workload's shapes.
BLOCK_BY_NAME = {"llama3_8b_block": BY_NAME["llama3_8b_mlp"]}


# ----------------------------------------------------------------------------- cross-entropy

CE_IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class CEConfig:
    """Cross-entropy over a vocabulary of V logits per token.

    logit_scale multiplies the logits (Cohere's logit scaling); softcap > 0
    applies c * tanh(t / c) after it (Gemma 2's final-logit softcapping).
    The raw logits are drawn with std `z_std`."""
    name: str
    N: int
    V: int
    logit_scale: float = 1.0
    softcap: float = 0.0
    z_std: float = 2.0
    ignore_frac: float = 0.03
    index: int = 70

    @property
    def seed(self) -> int:
        return 1234 + self.index

    def bytes_fwd(self) -> int:
        """Algorithmic HBM bytes of the forward: the logits read once."""
        return 2 * self.N * self.V

    def bytes_bwd(self) -> int:
        """Backward: the logits read once, their gradient written once."""
        return 4 * self.N * self.V


CE_CONFIGS = (
    CEConfig("ce_tiny", 37, 1003, 1.0, 0.0, index=70),
    CEConfig("ce_tiny_softcap", 45, 2051, 1.0, 30.0, z_std=10.0, index=71),
    CEConfig("ce_tiny_scale", 29, 777, 0.0625, 0.0, z_std=32.0, index=72),
    CEConfig("gemma2_256k_ce", 4096, 256000, 1.0, 30.0, z_std=10.0, index=73),
    CEConfig("cohere_256k_ce", 4096, 256000, 0.0625, 0.0, z_std=32.0, index=74),
    CEConfig("llama3_128k_ce", 4096, 128256, 1.0, 0.0, index=75),
    CEConfig("gemma2_256k_ce_1k", 1024, 256000, 1.0, 30.0, z_std=10.0, index=76),  # 1024 tokens: profiling size
)
CE_BY_NAME = {c.name: c for c in CE_CONFIGS}


def custom_ce(N, V, logit_scale=1.0, softcap=0.0, z_std=2.0, ignore_frac=0.03, seed_index=80,
              name="custom_ce") -> CEConfig:
    return CEConfig(name, N, V, logit_scale, softcap, z_std, ignore_frac, seed_index)


def make_ce_inputs(cfg: CEConfig) -> dict:
    """logits [N, V] bf16 bits ~ N(0, z_std^2) rounded to bf16; labels [N]
    int64 uniform in [0, V), a fraction ignore_frac of them replaced by
    CE_IGNORE_INDEX; dloss [N] float32 ~ U(0.5, 1.5) / N (a per-row upstream
    gradient that is not uniform, so a row mix-up shows).  One PCG64
    generator, seed 1234 + index, drawn in this order; the logits are drawn
    and rounded in blocks of rows so the float32 copy of a 256K vocabulary
    never exists whole."""
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    N, V = cfg.N, cfg.V
    z = np.empty((N, V), dtype=np.uint16)
    step = max(1, (1 << 24) // V)
    for r0 in range(0, N, step):
        r1 = min(N, r0 + step)
        blk = rng.standard_normal((r1 - r0, V), dtype=np.float32)
        blk *= np.float32(cfg.z_std)
        z[r0:r1] = f32_to_bf16_bits(blk)
    labels = rng.integers(0, V, size=N, dtype=np.int64)
    ignore = rng.random(N) < cfg.ignore_frac
    labels[ignore] = CE_IGNORE_INDEX
    dloss = (rng.uniform(0.5, 1.5, size=N) / N).astype(np.float32)
    return {"logits": z, "labels": labels, "dloss": dloss}
