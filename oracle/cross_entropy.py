"""fp64 CPU oracle of the chunked cross-entropy loss with logit scaling and
softcapping.

TEST INFRASTRUCTURE ONLY (tests/, bench.py's CPU legs); shares no code with
the CUDA path.

What it follows: "Unsloth 深度分析报告" (nightvoyager.top), section
核心价值提炼 / 创新之处, item 分块 Triton Cross Entropy Loss: the
cross-entropy loss of a very large vocabulary (256K) is computed chunk by
chunk, relying on logsumexp being separable over a partition of the
vocabulary, and it supports softcapping (Gemma 2) and logit scaling
(Cohere).  The same report's 可复用的模式与技巧 names the chunked-logsumexp
pattern for vocabularies above 65536 entries.  The pages print no formula; the
plain definitions, per row z of logits [V] with label y:

    t   = s * z                          logit scaling (s = logit_scale)
    t   = c * tanh(t / c)   if c > 0     softcapping (c = softcap)
    lse = log sum_j exp(t_j)
        = log sum_k exp(lse_k)           lse_k over the k-th vocabulary chunk
    loss = lse - t_y                     0 for a row whose y == ignore_index

and the chain rule for an upstream gradient dloss of the row:

    dz_j = dloss * (exp(t_j - lse) - [j == y]) * dt_j/dz_j,
    dt/dz = s                (no softcap)
          = s * (1 - (t/c)^2) (softcap: the derivative of c * tanh(s z / c))

with dz = 0 for ignored rows.  float64 throughout, from the exact bf16 input
values.
"""
from __future__ import annotations

import numpy as np

IGNORE_INDEX = -100
CHUNK = 65536  # vocabulary chunk of the forward (the pages' "above 65536 entries")


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def transform(z: np.ndarray, scale: float, softcap: float) -> np.ndarray:
    """t = s z, then c tanh(t / c) when softcap c > 0."""
    t = float(scale) * z
    if softcap > 0.0:
        t = float(softcap) * np.tanh(t / float(softcap))
    return t


def dtransform(t: np.ndarray, scale: float, softcap: float) -> np.ndarray:
    """dt/dz at the transformed logits t."""
    if softcap > 0.0:
        return float(scale) * (1.0 - (t / float(softcap)) ** 2)
    return np.full_like(t, float(scale))


def logsumexp_rows(t: np.ndarray) -> np.ndarray:
    """log sum_j exp(t_j) per row, with the row maximum factored out."""
    m = np.max(t, axis=1)
    return m + np.log(np.sum(np.exp(t - m[:, None]), axis=1))


def chunked_logsumexp(t: np.ndarray, chunk: int = CHUNK) -> np.ndarray:
    """The same quantity taken chunk by chunk over the vocabulary, then
    combined: log sum_k exp(lse_k)."""
    V = t.shape[1]
    parts = np.stack([logsumexp_rows(t[:, c0:c0 + chunk]) for c0 in range(0, V, chunk)], axis=1)
    return logsumexp_rows(parts)


def check_labels(labels: np.ndarray, V: int, ignore_index: int = IGNORE_INDEX) -> np.ndarray:
    labels = np.asarray(labels, dtype=np.int64)
    bad = (labels != ignore_index) & ((labels < 0) | (labels >= V))
    if np.any(bad):
        raise ValueError(f"labels outside [0, {V}) that are not ignore_index: {labels[bad][:4]}")
    return labels


def forward(z: np.ndarray, labels: np.ndarray, scale: float = 1.0, softcap: float = 0.0,
            ignore_index: int = IGNORE_INDEX, chunk: int = CHUNK):
    """Per-row (loss, lse) of logits z [N, V] (float64) and labels [N]."""
    N, V = z.shape
    labels = check_labels(labels, V, ignore_index)
    t = transform(z, scale, softcap)
    lse = chunked_logsumexp(t, chunk)
    valid = labels != ignore_index
    ty = np.zeros(N)
    ty[valid] = t[np.nonzero(valid)[0], labels[valid]]
    loss = np.where(valid, lse - ty, 0.0)
    return loss, lse


def backward(z: np.ndarray, labels: np.ndarray, lse: np.ndarray, dloss: np.ndarray, scale: float = 1.0,
             softcap: float = 0.0, ignore_index: int = IGNORE_INDEX) -> np.ndarray:
    """dz [N, V] for the upstream per-row gradient dloss [N]."""
    N, V = z.shape
    labels = check_labels(labels, V, ignore_index)
    t = transform(z, scale, softcap)
    g = np.exp(t - lse[:, None])
    valid = labels != ignore_index
    rows = np.nonzero(valid)[0]
    g[rows, labels[valid]] -= 1.0
    g *= dtransform(t, scale, softcap) * np.asarray(dloss, dtype=np.float64)[:, None]
    g[~valid] = 0.0
    return g


def rows(z_bits: np.ndarray, labels: np.ndarray, idx: np.ndarray, scale: float = 1.0, softcap: float = 0.0,
         dloss: np.ndarray | None = None, ignore_index: int = IGNORE_INDEX):
    """Loss, lse and (with dloss) dz of the rows `idx` of bf16 logits only:
    the sampled check of a full-size run."""
    z = bf16_to_f64(z_bits[idx])
    lab = np.asarray(labels)[idx]
    loss, lse = forward(z, lab, scale, softcap, ignore_index)
    dz = None if dloss is None else backward(z, lab, lse, np.asarray(dloss)[idx], scale, softcap, ignore_index)
    return loss, lse, dz
