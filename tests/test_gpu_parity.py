"""GPU parity: the sm_100a path through the C ABI against the fp64 CPU oracle.

Tolerance: per tensor, max|gpu - oracle| / max|oracle| <= 2e-2 for the bf16
outputs and gradients (fp32 accumulation).  The dequantisation of int4 and
FP8 frozen weights is compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu
TOL = 2e-2
GRADS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def run_gpu(inp, alpha, X_override=None):
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, alpha, dev)
    X = api.to_device_bf16(inp["X"] if X_override is None else X_override, dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    out, saved = api.forward(X, w)
    dX, grads = api.backward(X, w, saved, dOut)
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
    res = {"out": out, "g": saved.g, "u": saved.u, "dX": dX}
    res.update(grads)
    return {k: v.float().double().cpu().numpy() for k, v in res.items()}


def relerr(a, b):
    den = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (den if den > 0 else 1.0)


def assert_parity(got, ref, keys=("out", "dX") + GRADS, extra=(("g", "G"), ("u", "U")), tol=TOL):
    errs = {}
    for k in keys:
        errs[k] = relerr(got[k], ref[k])
    for gk, rk in extra:
        errs[gk] = relerr(got[gk], ref[rk])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"parity failures {bad}; all {errs}"
    return errs


SMALL_CASES = [
    synth.CONFIGS[0],                                            # tiny: d_ff = 704 = 5.5 tiles of 128
    synth.custom(300, 192, 320, 24, 8.0, seed_index=21),         # ragged N, r = 24 (padded MMA N)
    synth.custom(1, 64, 128, 8, 16.0, seed_index=22),            # a single token
    synth.custom(130, 136, 200, 16, 32.0, seed_index=23),        # K not a multiple of 64
    synth.custom(256, 256, 384, 128, 256.0, seed_index=24),      # maximum rank
    synth.custom(1000, 512, 1408, 64, 128.0, seed_index=25),     # several tiles in every dimension
]


@pytest.mark.parametrize("cfg", SMALL_CASES, ids=lambda c: f"N{c.N}_d{c.d}_dff{c.d_ff}_r{c.r}")
def test_parity_small(cfg):
    inp = synth.make_inputs(cfg)
    ref = oracle.forward_backward(inp, cfg.alpha)
    got = run_gpu(inp, cfg.alpha)
    assert_parity(got, ref)


def test_lora_delta_is_resolved():
    """The LoRA contribution (out(B) - out(B=0)) matches the oracle's delta,
    so the rank-r path cannot hide inside the 2e-2 band of the whole output."""
    cfg = synth.custom(512, 256, 704, 8, 16.0, seed_index=26)
    inp = synth.make_inputs(cfg)
    inp0 = synth.zero_B(inp)
    ref = oracle.forward_backward(inp, cfg.alpha)["out"] - oracle.forward_backward(inp0, cfg.alpha)["out"]
    got = run_gpu(inp, cfg.alpha)["out"] - run_gpu(inp0, cfg.alpha)["out"]
    assert relerr(got, ref) <= 5e-2


def test_zero_B_gives_frozen_mlp_and_zero_dA():
    cfg = synth.custom(384, 256, 512, 16, 16.0, seed_index=27)
    inp0 = synth.zero_B(synth.make_inputs(cfg))
    got = run_gpu(inp0, cfg.alpha)
    frozen = run_gpu(inp0, 0.0)
    assert np.array_equal(got["out"], frozen["out"])
    for k in ("dAg", "dAu", "dAd"):
        assert np.all(got[k] == 0.0), k
    ref = oracle.forward_backward(inp0, cfg.alpha)
    assert_parity(got, ref, keys=("out", "dX", "dBg", "dBu", "dBd"))


def test_deterministic_bits():
    cfg = synth.custom(640, 256, 512, 32, 32.0, seed_index=28)
    inp = synth.make_inputs(cfg)
    a = run_gpu(inp, cfg.alpha)
    b = run_gpu(inp, cfg.alpha)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_zero_input():
    cfg = synth.custom(128, 128, 256, 16, 16.0, seed_index=29)
    inp = synth.make_inputs(cfg)
    got = run_gpu(inp, cfg.alpha, X_override=np.zeros_like(inp["X"]))
    for k in ("out", "dX") + GRADS:
        assert np.all(got[k] == 0.0), k


# ----------------------------------------------------------------------------- int4


def test_dequant_bits_match_oracle():
    rng = np.random.default_rng(31)
    w = rng.standard_normal((96, 448)).astype(np.float32)
    w[5, 128:192] = 0.0
    q, sc = synth.quantize_int4(w)
    q[7, :8] = 0x88  # code -8 decodes too
    dev = torch.device("cuda:0")
    got = api.dequant_int4(torch.from_numpy(q).to(dev), torch.from_numpy(sc).to(dev))
    torch.cuda.synchronize()
    got_bits = got.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got_bits, oracle.dequant_int4(q, sc))


def test_dequant_bits_every_code_for_many_scales():
    """All 16 codes against finite scales of every kind: positive, negative,
    +-0, subnormal, the largest fp16."""
    rng = np.random.default_rng(36)
    sc = list(rng.uniform(-8, 8, 200).astype(np.float16))
    sc += [np.float16(x) for x in (0.0, -0.0, 6e-8, -6e-8, 1e-5, 65504.0, -65504.0, 1.0, 7.0, 0.1)]
    rows = len(sc)
    codes = np.tile(np.arange(-8, 8), (rows, 4))
    nib = (codes & 0xF).astype(np.uint8)
    q = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = np.array(sc, dtype=np.float16).reshape(rows, 1)
    dev = torch.device("cuda:0")
    got = api.dequant_int4(torch.from_numpy(q).to(dev), torch.from_numpy(scales).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), oracle.dequant_int4(q, scales))


def test_int4_path_matches_dequantised_bf16_path_bitwise_and_oracle():
    cfg = synth.custom(384, 256, 512, 16, 16.0, int4=True, seed_index=32)
    inp = synth.make_inputs(cfg)
    got4 = run_gpu(inp, cfg.alpha)
    deq = dict(inp)
    for k in ("Wg", "Wu", "Wd"):
        deq[k] = oracle.dequant_int4(inp[k + "_q"], inp[k + "_scale"])
        del deq[k + "_q"], deq[k + "_scale"]
    got16 = run_gpu(deq, cfg.alpha)
    for k in got4:
        assert np.array_equal(got4[k], got16[k]), k
    assert_parity(got4, oracle.forward_backward(inp, cfg.alpha))


# ----------------------------------------------------------------------------- FP8 (E4M3, fp32 scale per 64)


def same_bits_or_both_nan(got_bits, ref_bits):
    """bf16 bits equal, except that a NaN may carry any payload and sign."""
    f = lambda b: (np.asarray(b).astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    g, r = f(got_bits), f(ref_bits)
    nan = np.isnan(r)
    return np.array_equal(nan, np.isnan(g)) and np.array_equal(np.asarray(got_bits)[~nan], np.asarray(ref_bits)[~nan])


def test_fp8_dequant_bits_every_code_for_many_scales():
    """All 256 codes against fp32 scales of every kind: random over 82 decades,
    negative, +-0, subnormal, the largest finite, infinite and NaN."""
    rng = np.random.default_rng(37)
    sc = list(rng.uniform(-3, 3, 100).astype(np.float32)) + list((10.0 ** rng.uniform(-44, 38, 100)).astype(np.float32))
    sc += [0.0, -0.0, 1e-45, -1e-45, 1e-40, 2.0 ** -126, 3.4e38, -3.4e38, np.inf, -np.inf, np.nan, 1.0 / 448]
    sc = np.array(sc, dtype=np.float32)
    rows = len(sc)
    codes = np.tile(np.arange(256, dtype=np.uint8), (rows, 1))
    scales = np.repeat(sc[:, None], 4, axis=1)
    dev = torch.device("cuda:0")
    got = api.dequant_fp8(torch.from_numpy(codes).to(dev), torch.from_numpy(scales).to(dev))
    torch.cuda.synchronize()
    got_bits = got.view(torch.int16).cpu().numpy().view(np.uint16)
    assert same_bits_or_both_nan(got_bits, oracle.dequant_fp8(codes, scales))


def test_fp8_quantised_weight_dequantises_like_the_oracle():
    rng = np.random.default_rng(38)
    w = (rng.standard_normal((96, 448)) * 0.05).astype(np.float32)
    w[5, 128:192] = 0.0
    codes, scales = synth.quantize_fp8(w)
    dev = torch.device("cuda:0")
    got = api.dequant_fp8(torch.from_numpy(codes).view(torch.float8_e4m3fn).to(dev), torch.from_numpy(scales).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), oracle.dequant_fp8(codes, scales))


def dequantised_bf16_inputs(inp):
    deq = dict(inp)
    for k in ("Wg", "Wu", "Wd"):
        if k + "_f8" in inp:
            deq[k] = oracle.dequant_fp8(inp[k + "_f8"], inp[k + "_f8scale"])
            del deq[k + "_f8"], deq[k + "_f8scale"]
    return deq


@pytest.mark.parametrize("cfg", [synth.custom(384, 256, 512, 16, 16.0, seed_index=34, fp8=True),
                                 synth.custom(300, 192, 704, 24, 8.0, seed_index=35, fp8=True),   # ragged
                                 synth.custom(1000, 512, 1408, 64, 128.0, seed_index=36, fp8=True)],
                         ids=lambda c: f"N{c.N}_d{c.d}_dff{c.d_ff}_r{c.r}")
def test_fp8_path_matches_dequantised_bf16_path_bitwise_and_oracle(cfg):
    inp = synth.make_inputs(cfg)
    got8 = run_gpu(inp, cfg.alpha)
    got16 = run_gpu(dequantised_bf16_inputs(inp), cfg.alpha)
    for k in got8:
        assert np.array_equal(got8[k], got16[k]), k
    assert_parity(got8, oracle.forward_backward(inp, cfg.alpha))


# ----------------------------------------------------------------------------- autograd wrapper


def test_autograd_function_matches_api():
    cfg = synth.custom(256, 128, 256, 8, 8.0, seed_index=33)
    inp = synth.make_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, cfg.alpha, dev)
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        getattr(w, k).requires_grad_(True)
    X = api.to_device_bf16(inp["X"], dev).requires_grad_(True)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    out = api.LoRAMLPFunction.apply(X, w, w.Ag, w.Bg, w.Au, w.Bu, w.Ad, w.Bd)
    out.backward(dOut)
    ref = run_gpu(inp, cfg.alpha)
    assert np.array_equal(out.detach().float().double().cpu().numpy(), ref["out"])
    assert np.array_equal(X.grad.float().double().cpu().numpy(), ref["dX"])
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        assert np.array_equal(getattr(w, k).grad.float().double().cpu().numpy(), ref["d" + k]), k


def test_host_batch_trainer_back_to_back_steps():
    """Steps queued with no synchronisation in between: each step's gradient
    copy back must follow its own backward and finish before the step after
    next overwrites the device buffer, so the last two steps' host gradients
    equal the device-resident results bit for bit."""
    cfg_a = synth.custom(384, 256, 512, 16, 16.0, seed_index=36)
    inputs = [synth.make_inputs(synth.custom(384, 256, 512, 16, 16.0, seed_index=36 + i)) for i in range(3)]
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inputs[0], cfg_a.alpha, dev)
    host = [(torch.from_numpy(i["X"].view("int16")).view(torch.bfloat16).pin_memory(),
             torch.from_numpy(i["dOut"].view("int16")).view(torch.bfloat16).pin_memory()) for i in inputs]
    trainer = api.HostBatchTrainer(w, cfg_a.N, dev)
    order = [0, 1, 2, 1, 0]
    returned = []
    for i, b in enumerate(order):
        nxt = host[order[i + 1]] if i + 1 < len(order) else (None, None)
        returned.append(trainer.step(host[b][0], host[b][1], nxt[0], nxt[1]))
    trainer.finish()
    torch.cuda.synchronize()
    for i in (len(order) - 2, len(order) - 1):
        X = host[order[i]][0].to(dev)
        dOut = host[order[i]][1].to(dev)
        _, saved = api.forward(X, w)
        _, ref = api.backward(X, w, saved, dOut)
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(returned[i][k], ref[k].cpu()), (i, k)


def test_host_batch_trainer_matches_device_path():
    """Host batches through the overlapped-copy trainer give the same gradients
    as the device-resident calls, batch after batch."""
    cfg_a = synth.custom(512, 256, 512, 16, 16.0, seed_index=34)
    inp_a = synth.make_inputs(cfg_a)
    inp_b = synth.make_inputs(synth.custom(512, 256, 512, 16, 16.0, seed_index=35))
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp_a, cfg_a.alpha, dev)
    host = [(torch.from_numpy(i["X"].view("int16")).view(torch.bfloat16).pin_memory(),
             torch.from_numpy(i["dOut"].view("int16")).view(torch.bfloat16).pin_memory()) for i in (inp_a, inp_b)]
    trainer = api.HostBatchTrainer(w, cfg_a.N, dev)
    order = [0, 1, 0, 1]
    got = []
    for i, b in enumerate(order):
        nxt = host[order[i + 1]] if i + 1 < len(order) else (None, None)
        g = trainer.step(host[b][0], host[b][1], nxt[0], nxt[1])
        torch.cuda.synchronize()
        got.append({k: v.clone() for k, v in g.items()})
    for i, b in enumerate(order):
        X = host[b][0].to(dev)
        dOut = host[b][1].to(dev)
        _, saved = api.forward(X, w)
        _, ref = api.backward(X, w, saved, dOut)
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(got[i][k], ref[k].cpu()), (i, k)
