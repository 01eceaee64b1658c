"""Pins for the cross-entropy oracle: torch's library cross_entropy and
autograd in float64, central finite differences, the chunk-combination
identity of logsumexp, closed forms, and planted mistakes that the pins must
reject."""
import math

import numpy as np
import pytest
import torch

from oracle import cross_entropy as oce
from lora_fine_tuning_mlp_b200 import inputs as synth

IGN = oce.IGNORE_INDEX


def relerr(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def case(seed=3, N=6, V=50, z_std=3.0, ignore=(2,)):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((N, V)) * z_std
    labels = rng.integers(0, V, size=N)
    for i in ignore:
        labels[i] = IGN
    dloss = rng.uniform(0.5, 1.5, size=N)
    return z, labels, dloss


def torch_reference(z, labels, dloss, scale, softcap):
    """Loss per row and dz through torch: library cross_entropy on the
    transformed logits (torch.tanh for the softcap), autograd for dz."""
    tz = torch.from_numpy(z.copy()).requires_grad_(True)
    t = tz * scale
    if softcap > 0:
        t = softcap * torch.tanh(t / softcap)
    loss = torch.nn.functional.cross_entropy(t, torch.from_numpy(labels), reduction="none", ignore_index=IGN)
    (loss * torch.from_numpy(dloss)).sum().backward()
    return loss.detach().numpy(), tz.grad.numpy(), torch.logsumexp(t, dim=1).detach().numpy()


@pytest.mark.parametrize("scale,softcap", [(1.0, 0.0), (0.0625, 0.0), (1.0, 30.0), (0.7, 5.0)])
def test_matches_torch_cross_entropy_and_autograd(scale, softcap):
    z, labels, dloss = case(z_std=3.0 / scale if softcap == 0 else 8.0)
    loss, lse = oce.forward(z, labels, scale, softcap)
    dz = oce.backward(z, labels, lse, dloss, scale, softcap)
    tl, tdz, tlse = torch_reference(z, labels, dloss, scale, softcap)
    assert relerr(loss, tl) <= 1e-13
    assert relerr(lse, tlse) <= 1e-13
    assert relerr(dz, tdz) <= 1e-12


@pytest.mark.parametrize("scale,softcap", [(1.0, 0.0), (0.5, 0.0), (1.3, 4.0)])
def test_central_differences(scale, softcap):
    z, labels, dloss = case(seed=7, N=3, V=7, z_std=2.0, ignore=(1,))
    loss, lse = oce.forward(z, labels, scale, softcap)
    dz = oce.backward(z, labels, lse, dloss, scale, softcap)
    fd = np.zeros_like(z)
    for idx in np.ndindex(*z.shape):
        zp, zm = z.copy(), z.copy()
        zp[idx] += 1e-6
        zm[idx] -= 1e-6
        lp = float(np.sum(dloss * oce.forward(zp, labels, scale, softcap)[0]))
        lm = float(np.sum(dloss * oce.forward(zm, labels, scale, softcap)[0]))
        fd[idx] = (lp - lm) / 2e-6
    assert relerr(fd, dz) <= 1e-6


@pytest.mark.parametrize("chunk", [1, 3, 16, 49, 50, 1000])
def test_chunked_logsumexp_equals_the_whole_row(chunk):
    rng = np.random.default_rng(11)
    t = rng.standard_normal((5, 50)) * 20.0
    whole = np.log(np.sum(np.exp(t - t.max(axis=1, keepdims=True)), axis=1)) + t.max(axis=1)
    assert relerr(oce.chunked_logsumexp(t, chunk), whole) <= 1e-14


def test_closed_forms_and_invariances():
    V = 1000
    z = np.full((3, V), 1.7)
    labels = np.array([5, 999, IGN])
    loss, lse = oce.forward(z, labels)
    assert abs(loss[0] - math.log(V)) <= 1e-12 and abs(loss[1] - math.log(V)) <= 1e-12
    assert loss[2] == 0.0
    # a dominant correct logit gives loss -> 0 and gradient -> 0
    z2 = np.zeros((1, 10))
    z2[0, 4] = 60.0
    l2, s2 = oce.forward(z2, np.array([4]))
    assert 0.0 <= l2[0] < 1e-24
    # shift invariance without softcap; gradient rows sum to zero
    zr, lab, dl = case(seed=5)
    l0, s0 = oce.forward(zr, lab, 0.8)
    l1, s1 = oce.forward(zr + 123.0 / 0.8, lab, 0.8)
    assert relerr(l1, l0) <= 1e-10
    dz = oce.backward(zr, lab, s0, dl, 0.8)
    assert np.max(np.abs(dz.sum(axis=1))) <= 1e-12
    assert np.all(dz[lab == IGN] == 0.0)
    # a softcap far above the logits is the identity
    lc, _ = oce.forward(zr, lab, 0.8, 1e9)
    assert relerr(lc, l0) <= 1e-9
    # softcap: sum_j dz_j / (dt/dz)_j = 0 (the softmax part sums to one)
    lcap, scap = oce.forward(zr, lab, 1.0, 2.5)
    dzc = oce.backward(zr, lab, scap, dl, 1.0, 2.5)
    t = oce.transform(zr, 1.0, 2.5)
    assert np.max(np.abs((dzc / oce.dtransform(t, 1.0, 2.5)).sum(axis=1))) <= 1e-12


def test_labels_out_of_range_are_rejected():
    z, labels, _ = case()
    labels[0] = z.shape[1]
    with pytest.raises(ValueError):
        oce.forward(z, labels)


def test_sampled_rows_match_the_full_evaluation():
    cfg = synth.CE_BY_NAME["ce_tiny_softcap"]
    inp = synth.make_ce_inputs(cfg)
    z = oce.bf16_to_f64(inp["logits"])
    loss, lse = oce.forward(z, inp["labels"], cfg.logit_scale, cfg.softcap)
    dz = oce.backward(z, inp["labels"], lse, inp["dloss"], cfg.logit_scale, cfg.softcap)
    idx = np.array([0, 7, 44])
    l2, s2, d2 = oce.rows(inp["logits"], inp["labels"], idx, cfg.logit_scale, cfg.softcap, inp["dloss"])
    assert np.array_equal(l2, loss[idx]) and np.array_equal(s2, lse[idx]) and np.array_equal(d2, dz[idx])


# ----------------------------------------------------------------------------- planted mistakes

def _fwd_sign(z, labels, scale=1.0, softcap=0.0):
    loss, lse = oce.forward(z, labels, scale, softcap)
    t = oce.transform(z, scale, softcap)
    valid = labels != IGN
    ty = np.zeros(len(labels))
    ty[valid] = t[np.nonzero(valid)[0], labels[valid]]
    return np.where(valid, lse + ty, 0.0), lse


def _bwd_no_chain(z, labels, lse, dloss, scale=1.0, softcap=0.0):
    t = oce.transform(z, scale, softcap)
    p = np.exp(t - lse[:, None])
    valid = labels != IGN
    p[np.nonzero(valid)[0], labels[valid]] -= 1.0
    p *= np.asarray(dloss)[:, None] * scale
    p[~valid] = 0.0
    return p  # drops the softcap factor (1 - (t/c)^2)


def _bwd_onehot_sign(z, labels, lse, dloss, scale=1.0, softcap=0.0):
    g = oce.backward(z, labels, lse, dloss, scale, softcap)
    t = oce.transform(z, scale, softcap)
    valid = labels != IGN
    rows = np.nonzero(valid)[0]
    g[rows, labels[valid]] += 2.0 * dloss[valid] * oce.dtransform(t, scale, softcap)[rows, labels[valid]]
    return g


def _bwd_dloss_unscaled(z, labels, lse, dloss, scale=1.0, softcap=0.0):
    return oce.backward(z, labels, lse, np.ones_like(dloss), scale, softcap)


def _fwd_scale_after_cap(z, labels, scale=1.0, softcap=0.0):
    t = z.copy()
    if softcap > 0:
        t = softcap * np.tanh(t / softcap)
    t = scale * t
    lse = oce.chunked_logsumexp(t)
    valid = labels != IGN
    ty = np.zeros(len(labels))
    ty[valid] = t[np.nonzero(valid)[0], labels[valid]]
    return np.where(valid, lse - ty, 0.0), lse


def pins_hold(fwd, bwd, scale=0.7, softcap=5.0):
    z, labels, dloss = case(z_std=6.0)
    loss, lse = fwd(z, labels, scale, softcap)
    dz = bwd(z, labels, lse, dloss, scale, softcap)
    tl, tdz, _ = torch_reference(z, labels, dloss, scale, softcap)
    return relerr(loss, tl) <= 1e-12 and relerr(dz, tdz) <= 1e-11


def test_unmodified_oracle_passes():
    assert pins_hold(oce.forward, oce.backward)


@pytest.mark.parametrize("fwd,bwd", [
    (_fwd_sign, oce.backward),
    (oce.forward, _bwd_no_chain),
    (oce.forward, _bwd_onehot_sign),
    (oce.forward, _bwd_dloss_unscaled),
    (_fwd_scale_after_cap, oce.backward),
], ids=["loss_sign", "softcap_chain_dropped", "onehot_sign", "dloss_dropped", "scale_after_softcap"])
def test_planted_mistakes_are_rejected(fwd, bwd):
    assert not pins_hold(fwd, bwd)
