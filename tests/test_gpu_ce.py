"""GPU parity of the chunked cross-entropy (include/lora_ce.h) against the
fp64 oracle, through the C ABI: whole-matrix comparisons on small and ragged
vocabularies, sampled rows of the 256K-vocabulary workload, and the edge
cases (one logit, chunk boundaries, padded rows, ignored rows, masked and
extreme logits, in-place gradient, determinism, a bad label).

Tolerances, from the arithmetic: loss and lse within 1e-4 + 1e-5 |ref|
(fp32 sums of up to 2^18 exponentials); each gradient element within
2^-8 |ref| (its bf16 rounding, doubled) + 1e-5 * dloss * s (the fp32 error
of exp(t - lse) near the label's 1); and max|diff| / max|ref| <= 2e-2 per
tensor, the bar of the other bf16 outputs."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth
from oracle import cross_entropy as oce

pytestmark = pytest.mark.gpu
IGN = synth.CE_IGNORE_INDEX


@pytest.fixture(scope="module", autouse=True)
def _built():
    libbuild.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)


def dev_logits(bits: np.ndarray, ld=None):
    """bf16 logits on the device in rows of ld elements (default: V rounded
    up to a multiple of 8, the row-stride rule), zero padding."""
    N, V = bits.shape
    ld = (V + 7) // 8 * 8 if ld is None else ld
    buf = torch.zeros((N, ld), dtype=torch.int16)
    buf[:, :V] = torch.from_numpy(bits.view(np.int16))
    full = buf.view(torch.bfloat16).cuda()
    return full[:, :V], full


def run(bits, labels, dloss, scale, cap, ld=None, inplace=False):
    z, full = dev_logits(bits, ld)
    lab = torch.from_numpy(np.asarray(labels, dtype=np.int64)).cuda()
    dl = torch.from_numpy(np.asarray(dloss, dtype=np.float32)).cuda()
    loss, lse = api.ce_forward(z, lab, logit_scale=scale, softcap=cap, ignore_index=IGN)
    dz = api.ce_backward(z, lab, lse, dl, logit_scale=scale, softcap=cap, ignore_index=IGN, inplace=inplace)
    torch.cuda.synchronize()
    return (loss.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
            dz.float().cpu().numpy().astype(np.float64), full)


def check(bits, labels, dloss, scale, cap, loss, lse, dz):
    z = oce.bf16_to_f64(bits)
    rl, rs = oce.forward(z, labels, scale, cap, IGN)
    rd = oce.backward(z, labels, rs, dloss, scale, cap, IGN)
    assert np.all(np.abs(loss - rl) <= 1e-4 + 1e-5 * np.abs(rl)), np.max(np.abs(loss - rl))
    valid = np.asarray(labels) != IGN
    assert np.all(np.abs(lse - rs)[valid] <= 1e-4 + 1e-5 * np.abs(rs[valid]))
    atol = 1e-5 * np.asarray(dloss, dtype=np.float64)[:, None] * abs(scale)
    bad = np.abs(dz - rd) > 2.0 ** -8 * np.abs(rd) + atol
    assert not np.any(bad), (np.argwhere(bad)[:4], dz[bad][:4], rd[bad][:4])
    assert np.max(np.abs(dz - rd)) <= 2e-2 * max(np.max(np.abs(rd)), 1e-30)
    assert np.all(dz[~valid] == 0.0)


@pytest.mark.parametrize("name", ["ce_tiny", "ce_tiny_softcap", "ce_tiny_scale"])
def test_workloads_match_oracle(name):
    cfg = synth.CE_BY_NAME[name]
    inp = synth.make_ce_inputs(cfg)
    out = run(inp["logits"], inp["labels"], inp["dloss"], cfg.logit_scale, cfg.softcap)
    check(inp["logits"], inp["labels"], inp["dloss"], cfg.logit_scale, cfg.softcap, *out[:3])


@pytest.mark.parametrize("N,V,ld,scale,cap", [
    (3, 1, 8, 1.0, 0.0),            # one logit per row
    (5, 8, 8, 1.0, 0.0),            # one 16-byte vector
    (4, 9, 16, 0.5, 0.0),           # a ragged tail and padded rows
    (3, 8192, 8192, 1.0, 30.0),     # exactly one tile
    (3, 8193, 8200, 1.0, 0.0),      # one logit into a second tile
    (2, 40000, 40000, 2.0, 15.0),   # five tiles, scale and softcap
    (2, 65536, 65536, 1.0, 0.0),    # exactly one chunk (eight tiles)
    (2, 65537, 65544, 0.5, 0.0),    # one logit into a second chunk
    (1, 140001, 140008, 1.0, 30.0), # one row, three chunks, ragged last tile
])
def test_shapes_and_chunk_boundaries(N, V, ld, scale, cap):
    cfg = synth.custom_ce(N, V, scale, cap, z_std=3.0 / scale if cap == 0 else 10.0, ignore_frac=0.0,
                          seed_index=90 + V % 7)
    inp = synth.make_ce_inputs(cfg)
    labels = inp["labels"].copy()
    labels[0] = V - 1
    if N > 1:
        labels[1] = 0
    loss, lse, dz, _ = run(inp["logits"], labels, inp["dloss"], scale, cap, ld=ld)
    check(inp["logits"], labels, inp["dloss"], scale, cap, loss, lse, dz)
    # in place over padded rows: the same gradient, columns past V left alone
    l2, s2, d2, full = run(inp["logits"], labels, inp["dloss"], scale, cap, ld=ld, inplace=True)
    assert np.array_equal(d2, dz) and np.array_equal(l2, loss)
    if ld > V:
        assert torch.all(full[:, V:].view(torch.int16) == 0)


def test_ignored_rows_masked_and_extreme_logits():
    rng = np.random.default_rng(17)
    N, V = 6, 3000
    z = rng.standard_normal((N, V)).astype(np.float32) * 3
    z[0, :] = 0.0
    z[1, 10] = 3.0e4            # one dominant logit (loss ~ 0 when labelled)
    z[2, :100] = -np.inf        # masked vocabulary entries
    z[3, :] = 1.0e4             # all huge: lse must not overflow
    bits = synth.f32_to_bf16_bits(z)
    labels = np.array([7, 10, 500, 2999, IGN, IGN])
    dloss = rng.uniform(0.5, 1.5, N).astype(np.float32)
    loss, lse, dz, _ = run(bits, labels, dloss, 1.0, 0.0)
    check(bits, labels, dloss, 1.0, 0.0, loss, lse, dz)
    assert loss[4] == 0.0 and loss[5] == 0.0 and np.all(dz[4:] == 0.0)


def test_inplace_gradient_and_determinism():
    cfg = synth.CE_BY_NAME["ce_tiny_softcap"]
    inp = synth.make_ce_inputs(cfg)
    a = run(inp["logits"], inp["labels"], inp["dloss"], cfg.logit_scale, cfg.softcap)
    b = run(inp["logits"], inp["labels"], inp["dloss"], cfg.logit_scale, cfg.softcap)
    c = run(inp["logits"], inp["labels"], inp["dloss"], cfg.logit_scale, cfg.softcap, inplace=True)
    for x, y in ((a, b), (a, c)):
        assert np.array_equal(x[0], y[0]) and np.array_equal(x[1], y[1]) and np.array_equal(x[2], y[2])


def test_bad_label_is_reported_without_fault():
    cfg = synth.CE_BY_NAME["ce_tiny"]
    inp = synth.make_ce_inputs(cfg)
    labels = inp["labels"].copy()
    labels[3] = cfg.V + 5
    labels[4] = -7
    assert _lib.ce_device_status(None) == 0
    loss, lse, dz, _ = run(inp["logits"], labels, inp["dloss"], 1.0, 0.0)
    assert np.isnan(loss[3]) and np.isnan(loss[4])
    assert _lib.ce_device_status(None) == _lib.ERR_INVALID_ARG
    assert _lib.ce_device_status(None) == 0            # read and cleared
    ok = np.ones(cfg.N, bool)
    ok[[3, 4]] = False
    z = oce.bf16_to_f64(inp["logits"][ok])
    rl, _ = oce.forward(z, labels[ok])
    assert np.all(np.abs(loss[ok] - rl) <= 1e-4 + 1e-5 * np.abs(rl))


def test_autograd_mean_loss():
    cfg = synth.CE_BY_NAME["ce_tiny_scale"]
    inp = synth.make_ce_inputs(cfg)
    z = dev_logits(inp["logits"])[0].requires_grad_(True)
    before = z.detach().clone()
    lab = torch.from_numpy(inp["labels"]).cuda()
    loss = api.CrossEntropyFunction.apply(z, lab, cfg.logit_scale, 0.0, IGN)
    loss.backward()
    zz = oce.bf16_to_f64(inp["logits"])
    rl, rs = oce.forward(zz, inp["labels"], cfg.logit_scale, 0.0)
    n = max(int(np.sum(inp["labels"] != IGN)), 1)
    assert abs(loss.item() - rl.sum() / n) <= 1e-4 + 1e-5 * abs(rl.sum() / n)
    rd = oce.backward(zz, inp["labels"], rs, np.full(cfg.N, 1.0 / n), cfg.logit_scale, 0.0)
    g = z.grad.float().cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g - rd)) <= 2e-2 * np.max(np.abs(rd))
    assert not np.any(np.abs(g - rd) > 2.0 ** -8 * np.abs(rd) + 1e-5 * cfg.logit_scale / n)
    # by default the gradient goes to its own buffer: the logits are untouched
    assert torch.equal(z.detach(), before)


@pytest.mark.parametrize("reduction", ["sum", "mean"])
def test_reduced_loss_and_gradient_in_the_library(reduction):
    cfg = synth.CE_BY_NAME["ce_tiny_softcap"]
    inp = synth.make_ce_inputs(cfg)
    z, _ = dev_logits(inp["logits"])
    lab = torch.from_numpy(inp["labels"]).cuda()
    out, lse = api.ce_loss(z, lab, reduction=reduction, logit_scale=cfg.logit_scale, softcap=cfg.softcap,
                           ignore_index=IGN)
    dout = torch.tensor([0.75], dtype=torch.float32, device="cuda")
    dz = api.ce_backward_reduced(z, lab, lse, dout, out, logit_scale=cfg.logit_scale, softcap=cfg.softcap,
                                 ignore_index=IGN)
    torch.cuda.synchronize()
    zz = oce.bf16_to_f64(inp["logits"])
    rl, rs = oce.forward(zz, inp["labels"], cfg.logit_scale, cfg.softcap, IGN)
    n = max(int(np.sum(inp["labels"] != IGN)), 1)
    ref = rl.sum() / n if reduction == "mean" else rl.sum()
    factor = 1.0 / n if reduction == "mean" else 1.0
    got = out.cpu().numpy().astype(np.float64)
    assert abs(got[0] - ref) <= 1e-5 * abs(ref) + 1e-6, (got[0], ref)
    assert abs(got[1] - factor) <= 1e-7 * factor
    dl = np.full(cfg.N, 0.75 * factor)
    rd = oce.backward(zz, inp["labels"], rs, dl, cfg.logit_scale, cfg.softcap, IGN)
    d = dz.float().cpu().numpy().astype(np.float64)
    assert not np.any(np.abs(d - rd) > 2.0 ** -8 * np.abs(rd) + 1e-5 * dl[:, None] * cfg.logit_scale)
    assert np.max(np.abs(d - rd)) <= 2e-2 * np.max(np.abs(rd))
    # bitwise deterministic
    out2, _ = api.ce_loss(z, lab, reduction=reduction, logit_scale=cfg.logit_scale, softcap=cfg.softcap,
                          ignore_index=IGN)
    assert torch.equal(out, out2)


def test_inplace_gradient_is_opt_in_and_bumps_the_version():
    cfg = synth.custom_ce(33, 1000, seed_index=83)     # V a multiple of 8: dense rows
    inp = synth.make_ce_inputs(cfg)
    base = dev_logits(inp["logits"])[0].clone().requires_grad_(True)
    assert base.stride(0) == cfg.V
    z = base * 1.0          # a non-leaf the loss may overwrite
    v0 = z._version
    lab = torch.from_numpy(inp["labels"]).cuda()
    loss = api.CrossEntropyFunction.apply(z, lab, cfg.logit_scale, 0.0, IGN, True)
    loss.backward()
    assert z._version > v0
    zz = oce.bf16_to_f64(inp["logits"])
    rl, rs = oce.forward(zz, inp["labels"], cfg.logit_scale, 0.0)
    n = max(int(np.sum(inp["labels"] != IGN)), 1)
    rd = oce.backward(zz, inp["labels"], rs, np.full(cfg.N, 1.0 / n), cfg.logit_scale, 0.0)
    g = base.grad.float().cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g - rd)) <= 2e-2 * np.max(np.abs(rd))


@pytest.mark.parametrize("name", ["gemma2_256k_ce"])
def test_full_size_sampled_rows(name):
    cfg = synth.CE_BY_NAME[name]
    inp = synth.make_ce_inputs(cfg)
    z, _ = dev_logits(inp["logits"])
    lab = torch.from_numpy(inp["labels"]).cuda()
    dl = torch.from_numpy(inp["dloss"]).cuda()
    loss, lse = api.ce_forward(z, lab, logit_scale=cfg.logit_scale, softcap=cfg.softcap, ignore_index=IGN)
    dz = api.ce_backward(z, lab, lse, dl, logit_scale=cfg.logit_scale, softcap=cfg.softcap, ignore_index=IGN,
                         inplace=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    idx = np.sort(np.concatenate([[0, cfg.N - 1], rng.choice(cfg.N, 14, replace=False)]))
    idx = np.unique(idx)
    rl, rs, rd = oce.rows(inp["logits"], inp["labels"], idx, cfg.logit_scale, cfg.softcap, inp["dloss"], IGN)
    got_l = loss.cpu().numpy()[idx].astype(np.float64)
    got_s = lse.cpu().numpy()[idx].astype(np.float64)
    got_d = dz[torch.from_numpy(idx).cuda()].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got_l - rl) <= 1e-4 + 1e-5 * np.abs(rl))
    v = inp["labels"][idx] != IGN
    assert np.all(np.abs(got_s - rs)[v] <= 1e-4 + 1e-5 * np.abs(rs[v]))
    atol = 1e-5 * inp["dloss"][idx].astype(np.float64)[:, None] * cfg.logit_scale
    assert not np.any(np.abs(got_d - rd) > 2.0 ** -8 * np.abs(rd) + atol)
    # every row: the per-row loss is finite and the mean is near log V for these logits
    allv = inp["labels"] != IGN
    ll = loss.cpu().numpy()
    assert np.all(np.isfinite(ll)) and np.all(ll[~allv] == 0.0)
