"""GPU parity of RMSNorm and of the pre-norm block out = MLP(RMSNorm(X))
against the fp64 oracle.

Tolerance as everywhere: per tensor, max|gpu - oracle| / max|oracle| <= 2e-2
(bf16 storage, fp32 arithmetic); rstd (fp32, a scalar per row from an fp32
sum of squares) within 1e-5 relative.  The block must also equal, bit for
bit, the composition of its parts called one by one through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import rmsnorm as orn
from oracle import lora_mlp as om
from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu
TOL = 2e-2
EPS = synth.RMS_EPS
GRADS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def relerr(a, b):
    den = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (den if den > 0 else 1.0)


def np64(t):
    return t.float().double().cpu().numpy()


def run_block(inp, alpha, folded=False):
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    gamma = api.to_device_bf16(inp["gamma"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    if folded:
        w = api.fold_gamma(w, gamma)
    out, saved = api.block_forward(X, w, gamma, EPS, folded=folded)
    dX, grads = api.block_backward(X, w, gamma, saved, dOut, folded=folded)
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
    res = {"out": out, "g": saved.g, "u": saved.u, "dX": dX}
    res.update(grads)
    return {k: np64(v) for k, v in res.items()}


@pytest.mark.parametrize("N,d", [(1, 64), (37, 200), (300, 4096), (129, 8192)])
def test_rmsnorm_kernels_match_oracle(N, d):
    rng = np.random.default_rng(N + d)
    x32 = (rng.standard_normal((N, d)) * np.exp(rng.uniform(-3, 3, (N, 1)))).astype(np.float32)
    xb = synth.f32_to_bf16_bits(x32)
    gb = synth.f32_to_bf16_bits(rng.uniform(0.5, 1.5, d).astype(np.float32))
    db = synth.f32_to_bf16_bits(rng.standard_normal((N, d)).astype(np.float32))
    x, gamma, dy = (api.to_device_bf16(a) for a in (xb, gb, db))
    y, rstd = api.rmsnorm_forward(x, gamma, EPS)
    dx = api.rmsnorm_backward(x, gamma, rstd, dy)
    torch.cuda.synchronize()
    x64, g64, d64 = om.bf16_to_f64(xb), om.bf16_to_f64(gb), om.bf16_to_f64(db)
    y_ref, r_ref = orn.rmsnorm_forward(x64, g64, EPS)
    dx_ref = orn.rmsnorm_backward(x64, g64, r_ref, d64)
    assert np.max(np.abs(rstd.double().cpu().numpy() / r_ref - 1.0)) <= 1e-5
    assert relerr(np64(y), y_ref) <= TOL
    assert relerr(np64(dx), dx_ref) <= TOL
    assert torch.equal(api.rmsnorm_forward(x, gamma, EPS)[0], y)   # deterministic


SMALL = [
    synth.custom(512, 256, 704, 8, 16.0, seed_index=80),
    synth.custom(300, 192, 320, 24, 8.0, seed_index=81),
    synth.custom(1, 64, 128, 8, 16.0, seed_index=82),
    synth.custom(1000, 512, 1408, 64, 128.0, seed_index=83),
]


@pytest.mark.parametrize("folded", [False, True], ids=["norm_kernel", "gamma_folded"])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"N{c.N}_d{c.d}_dff{c.d_ff}_r{c.r}")
def test_block_parity_small(cfg, folded):
    inp = synth.make_block_inputs(cfg)
    ref = orn.block_forward_backward(inp, cfg.alpha, EPS)
    got = run_block(inp, cfg.alpha, folded)
    errs = {k: relerr(got[k], ref[k]) for k in ("out", "dX") + GRADS}
    errs["g"] = relerr(got["g"], ref["G"])
    errs["u"] = relerr(got["u"], ref["U"])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"parity failures {bad}; all {errs}"


def test_block_equals_its_parts_bitwise():
    """Also shows that the backward's recomputed normalised rows (from the
    cached rstd) are the forward's bit for bit: the adapter gradients of the
    block equal those of the MLP backward run on the forward's rows."""
    cfg = synth.custom(384, 256, 512, 16, 16.0, seed_index=84)
    inp = synth.make_block_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    gamma = api.to_device_bf16(inp["gamma"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    out, saved = api.block_forward(X, w, gamma, EPS)
    dX, grads = api.block_backward(X, w, gamma, saved, dOut)
    xn, rstd = api.rmsnorm_forward(X, gamma, EPS)
    out2, saved2 = api.forward(xn, w)
    dxn, grads2 = api.backward(xn, w, saved2, dOut)
    dX2 = api.rmsnorm_backward(X, gamma, rstd, dxn)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(saved.g, saved2.g) and torch.equal(saved.u, saved2.u)
    assert torch.equal(dX, dX2)
    for k in GRADS:
        assert torch.equal(grads[k], grads2[k]), k


def test_fold_gamma_is_the_rounded_column_product():
    """fold_gamma writes bf16_rne(W[j, c] * gamma[c]) (one fp32 product,
    exact for two bf16 factors, then one rounding) and shares the rest."""
    cfg = synth.custom(64, 192, 320, 8, 16.0, seed_index=86)
    inp = synth.make_block_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, cfg.alpha, dev)
    gamma = api.to_device_bf16(inp["gamma"], dev)
    wf = api.fold_gamma(w, gamma)
    torch.cuda.synchronize()
    for k in ("Wg", "Wu"):
        exact = om.bf16_to_f64(inp[k]) * om.bf16_to_f64(inp["gamma"])[None, :]
        want = om.f32_to_bf16_rne(exact.astype(np.float32))
        assert np.array_equal(getattr(wf, k).view(torch.int16).cpu().numpy().view(np.uint16), want), k
    assert wf.Wd is w.Wd and wf.Ag is w.Ag and wf.Bd is w.Bd


def test_folded_block_is_deterministic_and_near_the_unfused_block():
    cfg = synth.custom(1000, 512, 1408, 64, 128.0, seed_index=87)
    inp = synth.make_block_inputs(cfg)
    a = run_block(inp, cfg.alpha, folded=True)
    b = run_block(inp, cfg.alpha, folded=True)
    c = run_block(inp, cfg.alpha, folded=False)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
        assert relerr(a[k], c[k]) <= TOL, k


def test_rmsnorm_autograd_function_matches_oracle():
    """RMSNormFunction: forward y and backward dx (the gain is frozen) against
    the fp64 oracle."""
    rng = np.random.default_rng(61)
    N, d = 300, 1024
    x = (rng.standard_normal((N, d)) * rng.uniform(0.25, 4.0, (N, 1))).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, d).astype(np.float32)
    dy = rng.standard_normal((N, d)).astype(np.float32)
    xb, gb, dyb = (synth.f32_to_bf16_bits(a) for a in (x, gamma, dy))
    dev = torch.device("cuda:0")
    tx = api.to_device_bf16(xb, dev).requires_grad_(True)
    tg = api.to_device_bf16(gb, dev)
    y = api.RMSNormFunction.apply(tx, tg, EPS)
    y.backward(api.to_device_bf16(dyb, dev))
    x64, g64, dy64 = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in (xb, gb, dyb))
    ry, rstd = orn.rmsnorm_forward(x64, g64, EPS)
    rdx = orn.rmsnorm_backward(x64, g64, rstd, dy64)
    assert relerr(np64(y.detach()), ry) <= TOL
    assert relerr(np64(tx.grad), rdx) <= TOL


def test_block_autograd_function():
    cfg = synth.custom(200, 128, 256, 8, 16.0, seed_index=85)
    inp = synth.make_block_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, cfg.alpha, dev)
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        getattr(w, k).requires_grad_(True)
    X = api.to_device_bf16(inp["X"], dev).requires_grad_(True)
    gamma = api.to_device_bf16(inp["gamma"], dev)
    out = api.LoRAMLPBlockFunction.apply(X, w, gamma, EPS, w.Ag, w.Bg, w.Au, w.Bu, w.Ad, w.Bd)
    out.backward(api.to_device_bf16(inp["dOut"], dev))
    torch.cuda.synchronize()
    ref = orn.block_forward_backward(inp, cfg.alpha, EPS)
    assert relerr(np64(out.detach()), ref["out"]) <= TOL
    assert relerr(np64(X.grad), ref["dX"]) <= TOL
    for k in ("Ag", "Bd"):
        assert relerr(np64(getattr(w, k).grad), ref["d" + k]) <= TOL, k


@pytest.mark.slow
@pytest.mark.parametrize("folded", [False, True], ids=["norm_kernel", "gamma_folded"])
def test_block_full_size_sampled_rows(folded):
    cfg = synth.BY_NAME["llama3_8b_mlp"]
    inp = synth.make_block_inputs(cfg)
    got = run_block(inp, cfg.alpha, folded)
    torch.cuda.empty_cache()
    rng = np.random.default_rng(cfg.seed)
    rows = np.unique(np.concatenate([[0, cfg.N - 1], rng.choice(cfg.N, 30, replace=False)]))
    ref = orn.block_token_rows(inp, cfg.alpha, EPS, rows)
    errs = {k: relerr(got[g][rows], ref[k]) for g, k in (("out", "out"), ("g", "G"), ("u", "U"), ("dX", "dX"))}
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"{bad} (all {errs})"
