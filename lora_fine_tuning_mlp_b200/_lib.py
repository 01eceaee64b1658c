"""ctypes binding of liblora_mlp.so (include/lora_mlp.h, lora_linear.h, lora_rmsnorm.h, lora_ce.h).

Argument marshalling only: every step of the MLP runs in the library's CUDA
kernels.  Loading fails loudly if the shared library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblora_mlp.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_MISALIGNED = -3
ERR_WORKSPACE_TOO_SMALL = -4
ERR_UNSUPPORTED_ARCH = -5
ERR_CUDA = -6
ERR_DEVICE_TIMEOUT = -7

CE_REDUCTION_SUM = 1
CE_REDUCTION_MEAN = 2

WEIGHTS_BF16 = 0
WEIGHTS_INT4_B64 = 1
WEIGHTS_FP8_B64 = 2

WEIGHT_FIELDS = ("Wg", "Wu", "Wd", "Sg", "Su", "Sd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")
GRAD_FIELDS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")

# Every symbol include/lora_mlp.h, lora_linear.h, lora_rmsnorm.h and lora_ce.h declare.
SYMBOLS = (
    "lora_mlp_sizes",
    "lora_mlp_workspace_size",
    "lora_mlp_forward",
    "lora_mlp_backward",
    "lora_mlp_dequant_int4",
    "lora_mlp_dequant_fp8",
    "lora_mlp_device_status",
    "lora_mlp_check_pointer",
    "lora_mlp_strerror",
    "lora_mlp_timing_enable",
    "lora_mlp_timing_collect",
    "lora_mlp_launch_count",
    "lora_mlp_forward_noalloc",
    "lora_mlp_debug_force_timeout",
    "lora_linear_sizes",
    "lora_linear_forward",
    "lora_linear_backward",
    "lora_rmsnorm_forward",
    "lora_rmsnorm_backward",
    "lora_mlp_block_sizes",
    "lora_mlp_block_forward",
    "lora_mlp_block_backward",
    "lora_mlp_block_fold_gamma",
    "lora_mlp_block_forward_folded",
    "lora_mlp_block_backward_folded",
    "lora_ce_sizes",
    "lora_ce_forward",
    "lora_ce_backward",
    "lora_ce_forward_reduced",
    "lora_ce_backward_reduced",
    "lora_ce_device_status",
)


class Shape(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d", ctypes.c_int64), ("d_ff", ctypes.c_int64),
                ("r", ctypes.c_int64), ("alpha", ctypes.c_float), ("weight_format", ctypes.c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_FIELDS]


class LinShape(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d_in", ctypes.c_int64), ("d_out", ctypes.c_int64),
                ("r", ctypes.c_int64), ("alpha", ctypes.c_float), ("weight_format", ctypes.c_int32)]


class LinWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W", "S", "A", "B")]


class CEShape(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("V", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("logit_scale", ctypes.c_float), ("softcap", ctypes.c_float), ("ignore_index", ctypes.c_int64)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("ms", ctypes.c_float)]


class LoraMLPError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it first (python -c 'import __graft_entry__ as g; g.build()')")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
            L.lora_mlp_sizes.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                         ctypes.POINTER(sz)]
            L.lora_mlp_forward.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp, vp,
                                           vp, sz, vp]
            L.lora_mlp_backward.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp, vp,
                                            vp, ctypes.POINTER(Grads), vp, sz, vp]
            L.lora_mlp_dequant_int4.argtypes = [vp, vp, i64, i64, vp, vp]
            L.lora_mlp_dequant_fp8.argtypes = [vp, vp, i64, i64, vp, vp]
            L.lora_mlp_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
            L.lora_mlp_check_pointer.argtypes = [vp, sz]
            L.lora_mlp_strerror.argtypes = [ctypes.c_int]
            L.lora_mlp_strerror.restype = ctypes.c_char_p
            L.lora_mlp_timing_enable.argtypes = [ctypes.c_int]
            L.lora_mlp_timing_collect.argtypes = [ctypes.POINTER(KernelTime), ctypes.c_int,
                                                  ctypes.POINTER(ctypes.c_int)]
            L.lora_mlp_forward_noalloc.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp,
                                                   vp, vp]
            L.lora_mlp_debug_force_timeout.argtypes = [ctypes.c_int, i64]
            L.lora_mlp_debug_force_timeout.restype = ctypes.c_int
            L.lora_linear_sizes.argtypes = [ctypes.POINTER(LinShape), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                            ctypes.POINTER(sz)]
            L.lora_linear_forward.argtypes = [ctypes.POINTER(LinShape), ctypes.POINTER(LinWeights), vp, vp, vp,
                                              vp, sz, vp]
            L.lora_linear_backward.argtypes = [ctypes.POINTER(LinShape), ctypes.POINTER(LinWeights), vp, vp, vp,
                                               vp, vp, vp, vp, sz, vp]
            L.lora_rmsnorm_forward.argtypes = [i64, i64, ctypes.c_float, vp, vp, vp, vp, vp]
            L.lora_rmsnorm_backward.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp]
            L.lora_mlp_block_sizes.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                               ctypes.POINTER(sz)]
            L.lora_mlp_block_forward.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, ctypes.c_float,
                                                 vp, vp, vp, vp, vp, vp, sz, vp]
            L.lora_mlp_block_backward.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp,
                                                  vp, vp, vp, ctypes.POINTER(Grads), vp, sz, vp]
            L.lora_mlp_block_fold_gamma.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp]
            L.lora_mlp_block_forward_folded.argtypes = L.lora_mlp_block_forward.argtypes
            L.lora_mlp_block_backward_folded.argtypes = L.lora_mlp_block_backward.argtypes
            L.lora_ce_sizes.argtypes = [ctypes.POINTER(CEShape), ctypes.POINTER(sz)]
            L.lora_ce_forward.argtypes = [ctypes.POINTER(CEShape), vp, vp, vp, vp, vp, sz, vp]
            L.lora_ce_backward.argtypes = [ctypes.POINTER(CEShape), vp, vp, vp, vp, vp, vp]
            L.lora_ce_forward_reduced.argtypes = [ctypes.POINTER(CEShape), vp, vp, ctypes.c_int, vp, vp, vp, sz,
                                                  vp]
            L.lora_ce_backward_reduced.argtypes = [ctypes.POINTER(CEShape), vp, vp, vp, vp, vp, vp, vp]
            L.lora_mlp_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(sz), ctypes.POINTER(sz)]
            L.lora_ce_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
            L.lora_mlp_launch_count.argtypes = []
            L.lora_mlp_launch_count.restype = ctypes.c_int64
            for name in ("lora_mlp_sizes", "lora_mlp_forward", "lora_mlp_forward_noalloc", "lora_mlp_backward",
                         "lora_mlp_dequant_int4", "lora_mlp_dequant_fp8",
                         "lora_mlp_device_status", "lora_mlp_check_pointer", "lora_mlp_timing_enable",
                         "lora_mlp_timing_collect",
                         "lora_linear_sizes", "lora_linear_forward", "lora_linear_backward",
                         "lora_rmsnorm_forward", "lora_rmsnorm_backward", "lora_mlp_block_sizes",
                         "lora_mlp_block_forward", "lora_mlp_block_backward", "lora_ce_sizes",
                         "lora_ce_forward", "lora_ce_backward", "lora_ce_device_status",
                         "lora_ce_forward_reduced", "lora_ce_backward_reduced", "lora_mlp_workspace_size",
                         "lora_mlp_block_fold_gamma", "lora_mlp_block_forward_folded",
                         "lora_mlp_block_backward_folded"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def strerror(code: int) -> str:
    try:
        return lib().lora_mlp_strerror(code).decode()
    except ImportError:
        return "error"


def check(code: int, what: str) -> None:
    if code != OK:
        raise LoraMLPError(code, what)


def make_shape(N, d, d_ff, r, alpha, weight_format=WEIGHTS_BF16) -> Shape:
    return Shape(int(N), int(d), int(d_ff), int(r), float(alpha), int(weight_format))


def sizes(shape: Shape):
    f, b, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().lora_mlp_sizes(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(b), ctypes.byref(s)),
          "lora_mlp_sizes")
    return f.value, b.value, s.value


def workspace_size(shape: Shape):
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().lora_mlp_workspace_size(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(b)),
          "lora_mlp_workspace_size")
    return f.value, b.value


def forward(shape: Shape, weights: Weights, X, out, g, u, saved, workspace, workspace_bytes, stream) -> int:
    return lib().lora_mlp_forward(ctypes.byref(shape), ctypes.byref(weights), X, out, g, u, saved, workspace,
                                  workspace_bytes, stream)


def forward_noalloc(shape: Shape, weights: Weights, X, out, g, u, saved, stream) -> int:
    return lib().lora_mlp_forward_noalloc(ctypes.byref(shape), ctypes.byref(weights), X, out, g, u, saved, stream)


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def backward(shape: Shape, weights: Weights, X, g, u, saved, dOut, dX, grads: Grads, workspace,
             workspace_bytes, stream) -> int:
    return lib().lora_mlp_backward(ctypes.byref(shape), ctypes.byref(weights), X, g, u, saved, dOut, dX,
                                   ctypes.byref(grads), workspace, workspace_bytes, stream)


def dequant_int4(packed, scales, rows, cols, w_bf16, stream) -> int:
    return lib().lora_mlp_dequant_int4(packed, scales, int(rows), int(cols), w_bf16, stream)


def dequant_fp8(codes, scales, rows, cols, w_bf16, stream) -> int:
    return lib().lora_mlp_dequant_fp8(codes, scales, int(rows), int(cols), w_bf16, stream)


def check_pointer(ptr, alignment: int = 16) -> int:
    """The entry points' pointer check on its own (no launch): a LORA_MLP code."""
    return lib().lora_mlp_check_pointer(ptr, int(alignment))


def device_status(stream) -> int:
    v = ctypes.c_int(0)
    check(lib().lora_mlp_device_status(stream, ctypes.byref(v)), "lora_mlp_device_status")
    return v.value


def timing_enable(on: bool) -> None:
    check(lib().lora_mlp_timing_enable(1 if on else 0), "lora_mlp_timing_enable")


def timing_collect(max_records: int = 4096):
    buf = (KernelTime * max_records)()
    n = ctypes.c_int(0)
    check(lib().lora_mlp_timing_collect(buf, max_records, ctypes.byref(n)), "lora_mlp_timing_collect")
    return [(buf[i].name.decode(), float(buf[i].ms)) for i in range(min(n.value, max_records))]


def debug_force_timeout(enable: bool, wait_cycles: int = 0) -> None:
    check(lib().lora_mlp_debug_force_timeout(1 if enable else 0, int(wait_cycles)), "lora_mlp_debug_force_timeout")


def launch_count() -> int:
    return int(lib().lora_mlp_launch_count())


def make_lin_shape(N, d_in, d_out, r, alpha, weight_format=WEIGHTS_BF16) -> LinShape:
    return LinShape(int(N), int(d_in), int(d_out), int(r), float(alpha), int(weight_format))


def lin_sizes(shape: LinShape):
    f, b, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().lora_linear_sizes(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(b), ctypes.byref(s)),
          "lora_linear_sizes")
    return f.value, b.value, s.value


def lin_forward(shape: LinShape, weights: LinWeights, X, Y, saved, workspace, workspace_bytes, stream) -> int:
    return lib().lora_linear_forward(ctypes.byref(shape), ctypes.byref(weights), X, Y, saved, workspace,
                                     workspace_bytes, stream)


def lin_backward(shape: LinShape, weights: LinWeights, X, saved, dY, dX, dA, dB, workspace, workspace_bytes,
                 stream) -> int:
    return lib().lora_linear_backward(ctypes.byref(shape), ctypes.byref(weights), X, saved, dY, dX, dA, dB,
                                      workspace, workspace_bytes, stream)


def block_sizes(shape: Shape):
    f, b, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().lora_mlp_block_sizes(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(b), ctypes.byref(s)),
          "lora_mlp_block_sizes")
    return f.value, b.value, s.value


def block_forward(shape: Shape, weights: Weights, gamma, eps, X, out, g, u, saved, workspace, workspace_bytes,
                  stream) -> int:
    return lib().lora_mlp_block_forward(ctypes.byref(shape), ctypes.byref(weights), gamma, float(eps), X, out, g, u,
                                        saved, workspace, workspace_bytes, stream)


def block_backward(shape: Shape, weights: Weights, gamma, X, g, u, saved, dOut, dX, grads: Grads, workspace,
                   workspace_bytes, stream) -> int:
    return lib().lora_mlp_block_backward(ctypes.byref(shape), ctypes.byref(weights), gamma, X, g, u, saved, dOut,
                                         dX, ctypes.byref(grads), workspace, workspace_bytes, stream)


def block_fold_gamma(shape: Shape, weights: Weights, gamma, Wg_folded, Wu_folded, stream) -> int:
    return lib().lora_mlp_block_fold_gamma(ctypes.byref(shape), ctypes.byref(weights), gamma, Wg_folded, Wu_folded,
                                           stream)


def block_forward_folded(shape: Shape, weights: Weights, gamma, eps, X, out, g, u, saved, workspace,
                         workspace_bytes, stream) -> int:
    return lib().lora_mlp_block_forward_folded(ctypes.byref(shape), ctypes.byref(weights), gamma, float(eps), X, out,
                                               g, u, saved, workspace, workspace_bytes, stream)


def block_backward_folded(shape: Shape, weights: Weights, gamma, X, g, u, saved, dOut, dX, grads: Grads, workspace,
                          workspace_bytes, stream) -> int:
    return lib().lora_mlp_block_backward_folded(ctypes.byref(shape), ctypes.byref(weights), gamma, X, g, u, saved,
                                                dOut, dX, ctypes.byref(grads), workspace, workspace_bytes, stream)


def rmsnorm_forward(N, d, eps, x, gamma, y, rstd, stream) -> int:
    return lib().lora_rmsnorm_forward(int(N), int(d), float(eps), x, gamma, y, rstd, stream)


def rmsnorm_backward(N, d, x, gamma, rstd, dy, dx, stream) -> int:
    return lib().lora_rmsnorm_backward(int(N), int(d), x, gamma, rstd, dy, dx, stream)


def make_ce_shape(N, V, ld=None, logit_scale=1.0, softcap=0.0, ignore_index=-100) -> CEShape:
    return CEShape(int(N), int(V), int(V if ld is None else ld), float(logit_scale), float(softcap),
                   int(ignore_index))


def ce_sizes(shape: CEShape) -> int:
    ws = ctypes.c_size_t()
    check(lib().lora_ce_sizes(ctypes.byref(shape), ctypes.byref(ws)), "lora_ce_sizes")
    return ws.value


def ce_forward(shape: CEShape, logits, labels, loss, lse, workspace, workspace_bytes, stream) -> int:
    return lib().lora_ce_forward(ctypes.byref(shape), logits, labels, loss, lse, workspace, workspace_bytes, stream)


def ce_backward(shape: CEShape, logits, labels, lse, dloss, dlogits, stream) -> int:
    return lib().lora_ce_backward(ctypes.byref(shape), logits, labels, lse, dloss, dlogits, stream)


def ce_forward_reduced(shape: CEShape, logits, labels, reduction, out, lse, workspace, workspace_bytes,
                       stream) -> int:
    return lib().lora_ce_forward_reduced(ctypes.byref(shape), logits, labels, int(reduction), out, lse, workspace,
                                         workspace_bytes, stream)


def ce_backward_reduced(shape: CEShape, logits, labels, lse, dout, fwd_out, dlogits, stream) -> int:
    return lib().lora_ce_backward_reduced(ctypes.byref(shape), logits, labels, lse, dout, fwd_out, dlogits, stream)


def ce_device_status(stream) -> int:
    st = ctypes.c_int(0)
    check(lib().lora_ce_device_status(stream, ctypes.byref(st)), "lora_ce_device_status")
    return st.value
