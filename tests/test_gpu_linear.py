"""GPU parity of the LoRA linear (include/lora_linear.h) against its fp64 oracle.

Tolerance as for the MLP: per tensor, max|gpu - oracle| / max|oracle| <= 2e-2
(bf16 storage, fp32 accumulation).  Small and ragged shapes are compared on
every output; the attention-projection shapes (Llama-3-8B q and k
projections, 4096 tokens) are compared on every output too, since their
oracle takes a few seconds."""
import numpy as np
import pytest
import torch

from oracle import lora_linear as olin
from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu
TOL = 2e-2
KEYS = ("Y", "dX", "dA", "dB")


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def cfg_of(N, d_in, d_out, r, alpha, idx, int4=False, fp8=False):
    return synth.LinearConfig(f"lin_{N}_{d_in}_{d_out}_{r}", N, d_in, d_out, r, float(alpha), int4=int4,
                              index=idx, fp8=fp8)


def run_gpu(inp, alpha, w=None, X_override=None):
    dev = torch.device("cuda:0")
    w = api.linear_weights_from_host(inp, alpha, dev) if w is None else w
    X = api.to_device_bf16(inp["X"] if X_override is None else X_override, dev)
    dY = api.to_device_bf16(inp["dY"], dev)
    Y, saved = api.linear_forward(X, w)
    dX, dA, dB = api.linear_backward(X, w, saved, dY)
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
    return {k: v.float().double().cpu().numpy() for k, v in (("Y", Y), ("dX", dX), ("dA", dA), ("dB", dB))}


def relerr(a, b):
    den = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (den if den > 0 else 1.0)


def assert_parity(got, ref, keys=KEYS, tol=TOL):
    errs = {k: relerr(got[k], ref[k]) for k in keys}
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"parity failures {bad}; all {errs}"
    return errs


SMALL = [
    synth.LINEAR_BY_NAME["linear_tiny"],      # ragged N (300), d_out 320 = 1.25 CTA-pair tiles
    cfg_of(1, 64, 128, 8, 16.0, 60),          # a single token
    cfg_of(130, 136, 200, 16, 32.0, 61),      # K not a multiple of 64 in either direction
    cfg_of(256, 256, 384, 128, 256.0, 62),    # maximum rank
    cfg_of(1000, 512, 1408, 24, 48.0, 63),    # several tiles everywhere, r = 24 (padded MMA N)
    cfg_of(777, 1024, 264, 64, 16.0, 64),     # d_out narrower than one tile pair
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_linear_parity_small(cfg):
    inp = synth.make_linear_inputs(cfg)
    ref = olin.forward_backward(inp, cfg.alpha)
    assert_parity(run_gpu(inp, cfg.alpha), ref)


def test_linear_lora_delta_is_resolved():
    """Y(B) - Y(B=0) against the oracle's delta: the rank-r path cannot hide
    inside the tolerance band of the whole output.  Both GPU outputs are
    rounded to bf16 (relative half-ulp 2^-9), so their difference carries up
    to 2^-8 max|Y| of rounding on top of the 2e-2 band of the delta itself."""
    cfg = cfg_of(512, 256, 640, 16, 64.0, 65)
    inp = synth.make_linear_inputs(cfg)
    inp0 = dict(inp, B=np.zeros_like(inp["B"]))
    Yref = olin.forward_backward(inp, cfg.alpha)["Y"]
    ref = Yref - olin.forward_backward(inp0, cfg.alpha)["Y"]
    got = run_gpu(inp, cfg.alpha)["Y"] - run_gpu(inp0, cfg.alpha)["Y"]
    bound = 2.0 ** -8 * np.max(np.abs(Yref)) + TOL * np.max(np.abs(ref))
    assert np.max(np.abs(got - ref)) <= bound
    assert np.max(np.abs(ref)) >= 10 * 2.0 ** -8 * np.max(np.abs(Yref))  # the delta is well resolved


def test_linear_zero_B_and_determinism():
    cfg = cfg_of(384, 256, 512, 16, 16.0, 66)
    inp = synth.make_linear_inputs(cfg)
    inp0 = dict(inp, B=np.zeros_like(inp["B"]))
    got = run_gpu(inp0, cfg.alpha)
    assert np.array_equal(got["Y"], run_gpu(inp0, 0.0)["Y"])
    assert np.all(got["dA"] == 0.0)
    assert_parity(got, olin.forward_backward(inp0, cfg.alpha), keys=("Y", "dX", "dB"))
    a, b = run_gpu(inp, cfg.alpha), run_gpu(inp, cfg.alpha)
    for k in KEYS:
        assert np.array_equal(a[k], b[k]), k


def test_linear_int4_matches_dequantised_bf16_bitwise_and_oracle():
    cfg = cfg_of(640, 512, 384, 16, 16.0, 67, int4=True)
    inp = synth.make_linear_inputs(cfg)
    dev = torch.device("cuda:0")
    w4 = api.linear_weights_from_host(inp, cfg.alpha, dev)
    Wbf = api.dequant_int4(w4.W, w4.S)
    wbf = api.LinearWeights(W=Wbf, A=w4.A, B=w4.B, alpha=cfg.alpha)
    g4 = run_gpu(inp, cfg.alpha, w=w4)
    gbf = run_gpu(inp, cfg.alpha, w=wbf)
    for k in KEYS:
        assert np.array_equal(g4[k], gbf[k]), k
    assert_parity(g4, olin.forward_backward(inp, cfg.alpha))


def test_linear_autograd_function():
    cfg = cfg_of(200, 128, 256, 8, 16.0, 68)
    inp = synth.make_linear_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.linear_weights_from_host(inp, cfg.alpha, dev)
    w.A.requires_grad_(True)
    w.B.requires_grad_(True)
    X = api.to_device_bf16(inp["X"], dev).requires_grad_(True)
    dY = api.to_device_bf16(inp["dY"], dev)
    Y = api.LoRALinearFunction.apply(X, w, w.A, w.B)
    Y.backward(dY)
    torch.cuda.synchronize()
    got = {k: v.detach().float().double().cpu().numpy()
           for k, v in (("Y", Y), ("dX", X.grad), ("dA", w.A.grad), ("dB", w.B.grad))}
    assert_parity(got, olin.forward_backward(inp, cfg.alpha))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama3_8b_qproj", "llama3_8b_kproj"])
def test_linear_full_size_every_output(name):
    cfg = synth.LINEAR_BY_NAME[name]
    inp = synth.make_linear_inputs(cfg)
    got = run_gpu(inp, cfg.alpha)
    torch.cuda.empty_cache()
    assert_parity(got, olin.forward_backward(inp, cfg.alpha))


@pytest.mark.parametrize("N,d_in,d_out", [(640, 512, 384), (300, 192, 328)])   # the second: d_out % 64 != 0
def test_linear_fp8_matches_dequantised_bf16_bitwise_and_oracle(N, d_in, d_out):
    cfg = cfg_of(N, d_in, d_out, 16, 16.0, 68, fp8=True)
    inp = synth.make_linear_inputs(cfg)
    dev = torch.device("cuda:0")
    w8 = api.linear_weights_from_host(inp, cfg.alpha, dev)
    Wbf = api.dequant_fp8(w8.W, w8.S)
    wbf = api.LinearWeights(W=Wbf, A=w8.A, B=w8.B, alpha=cfg.alpha)
    g8 = run_gpu(inp, cfg.alpha, w=w8)
    gbf = run_gpu(inp, cfg.alpha, w=wbf)
    for k in KEYS:
        assert np.array_equal(g8[k], gbf[k]), k
    assert_parity(g8, olin.forward_backward(inp, cfg.alpha))
