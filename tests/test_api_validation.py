"""The Python API refuses what its kernels cannot take, before any library
call: host (CPU) tensors and non-tensors.  On a machine without a GPU this is
also the check that the product path has no CPU fallback: every entry point
raises instead of computing."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_mlp_b200 import api

BF16 = torch.bfloat16


def cpu_mlp_weights(d=64, d_ff=128, r=8):
    z = lambda *s: torch.zeros(*s, dtype=BF16)  # noqa: E731
    return api.MLPWeights(Wg=z(d_ff, d), Wu=z(d_ff, d), Wd=z(d, d_ff), Ag=z(r, d), Bg=z(d_ff, r), Au=z(r, d),
                          Bu=z(d_ff, r), Ad=z(r, d_ff), Bd=z(d, r), alpha=16.0)


def test_mlp_forward_and_backward_refuse_host_tensors():
    w = cpu_mlp_weights()
    X = torch.zeros(4, 64, dtype=BF16)
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.forward(X, w)
    with pytest.raises(TypeError):
        api.forward(np.zeros((4, 64), dtype=np.float32), w)
    saved = api.Saved(torch.zeros(4, 128, dtype=BF16), torch.zeros(4, 128, dtype=BF16),
                      torch.zeros(256, dtype=torch.uint8))
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.backward(X, w, saved, torch.zeros(4, 64, dtype=BF16))


def test_other_entry_points_refuse_host_tensors():
    x = torch.zeros(4, 64, dtype=BF16)
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.rmsnorm_forward(x, torch.ones(64, dtype=BF16), 1e-5)
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.ce_forward(torch.zeros(4, 128, dtype=BF16), torch.zeros(4, dtype=torch.int64))
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.dequant_int4(torch.zeros(8, 32, dtype=torch.uint8), torch.zeros(8, 1, dtype=torch.float16))
    lw = api.LinearWeights(W=torch.zeros(64, 64, dtype=BF16), A=torch.zeros(8, 64, dtype=BF16),
                           B=torch.zeros(64, 8, dtype=BF16), alpha=16.0)
    with pytest.raises((ValueError, TypeError), match="CUDA"):
        api.linear_forward(x, lw)
