"""Failure detection without a GPU fault: every barrier wait in the library's
kernels is bounded.  The test hook makes each GEMM's epilogue wait on a
barrier that nothing signals, with a short limit; the kernels must give up,
report LORA_MLP_ERR_DEVICE_TIMEOUT through the status word, and leave the
CUDA context usable (a normal run afterwards matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu


def test_forced_wait_timeout_is_reported_and_the_context_survives():
    libbuild.build()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[0]
    inp = synth.make_inputs(cfg)
    w = api.weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    assert _lib.device_status(None) == 0
    _lib.debug_force_timeout(True, 20_000_000)  # about 10 ms at 2 GHz
    try:
        out, saved = api.forward(X, w)
        api.backward(X, w, saved, dOut)
        torch.cuda.synchronize()  # the kernels ended by themselves, without a CUDA error
    finally:
        _lib.debug_force_timeout(False)
    assert _lib.device_status(None) == _lib.ERR_DEVICE_TIMEOUT
    assert _lib.device_status(None) == 0  # reading clears it

    out, saved = api.forward(X, w)
    dX, grads = api.backward(X, w, saved, dOut)
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
    ref = oracle.forward_backward(inp, cfg.alpha)
    for name, t in (("out", out), ("dX", dX), *grads.items()):
        a = t.float().double().cpu().numpy()
        b = ref[name]
        assert np.max(np.abs(a - b)) / np.max(np.abs(b)) <= 2e-2, name
