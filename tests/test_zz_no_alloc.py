"""lora_mlp_forward_noalloc, the forward entry point that allocates nothing.

Callers that cannot allocate device memory themselves (a plugin inside a host
framework that owns all device memory, a latency-critical loop that cannot
afford cudaMalloc's device synchronisation, a deployment whose memory is
budgeted up front) get the forward pass with its scratch in a fixed array
inside the library.  Here it is called through the C ABI, twice in a row, and
its outputs are checked against lora_mlp_forward's on the same inputs, with
the tolerance the parity tests use.  The file sorts last so that a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


def relerr(a, b):
    a = a.float().double().cpu().numpy()
    b = b.float().double().cpu().numpy()
    den = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (den if den > 0 else 1.0)


@pytest.mark.parametrize("cfg", [synth.CONFIGS[0], synth.custom(1000, 512, 1408, 32, 64.0, seed_index=41),
                                 synth.custom(512, 256, 704, 8, 16.0, int4=True, seed_index=42)],
                         ids=lambda c: f"N{c.N}_d{c.d}_dff{c.d_ff}_r{c.r}" + ("_int4" if c.int4 else ""))
def test_noalloc_forward_matches_forward_on_two_calls(cfg):
    libbuild.build()
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(cfg)
    w = api.weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    shape = w.shape(cfg.N)
    fws, _, svs = _lib.sizes(shape)
    assert fws <= _lib.NOALLOC_SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    ref_out, ref_saved = api.forward(X, w)
    ref_dX, ref_grads = api.backward(X, w, ref_saved, dOut)

    for call in range(2):
        out = torch.full((cfg.N, cfg.d), float("nan"), dtype=torch.bfloat16, device=dev)
        g = torch.full((cfg.N, cfg.d_ff), float("nan"), dtype=torch.bfloat16, device=dev)
        u = torch.full_like(g, float("nan"))
        saved = torch.zeros(max(svs, 256), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info(dev)[0]
        rc = _lib.forward_noalloc(shape, w.c_struct(), P(X), P(out), P(g), P(u), P(saved), stream)
        assert rc == _lib.OK, _lib.strerror(rc)
        torch.cuda.synchronize()
        if call == 1:
            # the first call on a device may load the module that holds the
            # array; from then on a call takes no device memory at all
            assert torch.cuda.mem_get_info(dev)[0] == free0
        assert relerr(out, ref_out) <= TOL, call
        assert relerr(g, ref_saved.g) <= TOL, call
        assert relerr(u, ref_saved.u) <= TOL, call
        # what it saved drives the regular backward to the same gradients
        dX, grads = api.backward(X, w, api.Saved(g, u, saved), dOut)
        torch.cuda.synchronize()
        assert relerr(dX, ref_dX) <= TOL, call
        for k, v in grads.items():
            assert relerr(v, ref_grads[k]) <= TOL, (call, k)
    assert _lib.device_status(None) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    libbuild.build()
    shape = _lib.make_shape(4096, 4096, 14336, 16, 16.0)
    fws, _, _ = _lib.sizes(shape)
    assert fws > _lib.NOALLOC_SCRATCH_BYTES
    FAKE = 0x10000
    w = _lib.Weights(*[None if n in ("Sg", "Su", "Sd") else FAKE for n in _lib.WEIGHT_FIELDS])
    rc = _lib.forward_noalloc(shape, w, FAKE, FAKE, FAKE, FAKE, FAKE, None)
    assert rc == _lib.ERR_WORKSPACE_TOO_SMALL
