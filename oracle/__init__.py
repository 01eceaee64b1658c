"""CPU oracle (fp64) for the fused LoRA + SwiGLU MLP.

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm may import it; the product path never does.
"""
from .lora_mlp import (  # noqa: F401
    backward,
    bf16_to_f64,
    dequant_fp8,
    dequant_int4,
    e4m3_to_f64,
    f32_to_bf16_rne,
    forward,
    forward_backward,
    sigmoid,
    token_rows,
    up_gate_feature_grads,
    weights_f64,
)
from . import lora_linear  # noqa: F401,E402
from . import rmsnorm  # noqa: F401,E402
from . import cross_entropy  # noqa: F401,E402
