"""Fused LoRA + SwiGLU MLP for NVIDIA B200 (sm_100a).

The compute lives in liblora_mlp.so (C ABI: include/lora_mlp.h); `api` wraps
it for PyTorch tensors.  Importing this package does not load the CUDA
library; the first call does, and fails loudly if it is missing.
"""
import os

PACKAGE_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PACKAGE_DIR, "liblora_mlp.so")
