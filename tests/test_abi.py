"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol the header declares, sizes its buffers, and rejects bad
arguments with the documented codes before touching the device."""
import ctypes
import os
import re

import pytest

from lora_fine_tuning_mlp_b200 import _lib
from lora_fine_tuning_mlp_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("lora_mlp.h", "lora_linear.h", "lora_rmsnorm.h", "lora_ce.h")]


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.lib()


def header_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_(?:mlp|linear|rmsnorm|ce)_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert header_symbols() == sorted(_lib.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in header_symbols():
        assert hasattr(L, name), name


def test_strerror_codes(L):
    for code in range(0, -8, -1):
        assert _lib.strerror(code) not in ("", "unknown error")
    assert _lib.strerror(-99) == "unknown error"


def shape(N=512, d=256, d_ff=704, r=8, alpha=16.0, fmt=0):
    return _lib.make_shape(N, d, d_ff, r, alpha, fmt)


def test_sizes_are_positive_and_grow_with_N(L):
    f1, b1, s1 = _lib.sizes(shape(N=512))
    f2, b2, s2 = _lib.sizes(shape(N=4096))
    assert 0 < f1 < f2 and 0 < b1 < b2 and 0 < s1 < s2
    # the saved rank-r buffer holds three bf16 [r, N] tiles (N padded to 8)
    assert s1 >= 3 * 8 * 512 * 2
    # backward keeps dg, du and h in its workspace
    assert b1 >= 3 * 512 * 704 * 2


def test_one_pass_adapter_gradient_buffers_only_for_ranks_up_to_32(L):
    """Ranks <= 32 run the adapter-gradient reductions in one pass and keep
    their fp32 partial sums in the backward workspace: at least one token
    range's dB part (3 x d_ff x r) and one feature range's T part (N x 2r);
    rank 40 (> 32) keeps the split-K form, whose workspace is smaller than
    rank 32's although its rank is larger."""
    N, d, dff = 4096, 4096, 14336
    bw = {r: _lib.sizes(shape(N=N, d=d, d_ff=dff, r=r))[1] for r in (16, 32, 40)}
    for r in (16, 32):
        assert bw[r] >= 3 * N * dff * 2 + 4 * (3 * dff * r + N * 2 * r)
    assert bw[40] < bw[32]


def test_int4_workspace_holds_no_dequantised_weight(L):
    with pytest.raises(_lib.LoraMLPError) as e:
        _lib.sizes(shape(d=256, d_ff=712, fmt=1))   # 712 is not a multiple of 64
    assert e.value.code == _lib.ERR_UNSUPPORTED_SHAPE
    # int4 weights are dequantised inside the GEMMs: the scratch is the bf16
    # path's plus the three weights' block scales in transposed order
    for kw in (dict(d=256, d_ff=768), dict(N=4096, d=4096, d_ff=14336, r=16)):
        f4, b4, s4 = _lib.sizes(shape(fmt=1, **kw))
        f0, b0, s0 = _lib.sizes(shape(fmt=0, **kw))
        scales = 3 * (kw["d"] * kw["d_ff"] // 64 * 2 + 256)
        assert s4 == s0 and 0 < f4 - f0 <= scales and 0 < b4 - b0 <= scales
        assert f4 - f0 < kw["d"] * kw["d_ff"] * 2 // 16     # far below one bf16 weight
    lf = _lib.LinShape(4096, 4096, 1024, 16, 16.0, 1)
    lb = _lib.LinShape(4096, 4096, 1024, 16, 16.0, 0)
    (f4, b4, _), (f0, b0, _) = _lib.lin_sizes(lf), _lib.lin_sizes(lb)
    assert 0 < f4 - f0 <= 4096 * 1024 // 64 * 2 + 256 and 0 < b4 - b0 <= 4096 * 1024 // 64 * 2 + 256


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), _lib.ERR_INVALID_ARG),
    (dict(d=-8), _lib.ERR_INVALID_ARG),
    (dict(alpha=float("nan")), _lib.ERR_INVALID_ARG),
    (dict(alpha=float("inf")), _lib.ERR_INVALID_ARG),
    (dict(fmt=7), _lib.ERR_INVALID_ARG),
    (dict(d=260), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(d_ff=700), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(r=12), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(r=136), _lib.ERR_UNSUPPORTED_SHAPE),
])
def test_shape_validation(L, kw, code):
    sh = shape(**kw)
    f = ctypes.c_size_t()
    assert L.lora_mlp_sizes(ctypes.byref(sh), ctypes.byref(f), None, None) == code


FAKE = 0x10000  # a 16-byte-aligned non-null address: never dereferenced, validation fails first


def weights(**over):
    vals = {n: FAKE for n in _lib.WEIGHT_FIELDS}
    vals.update({"Sg": None, "Su": None, "Sd": None})
    vals.update(over)
    return _lib.Weights(*[vals[n] for n in _lib.WEIGHT_FIELDS])


def fwd(L, sh, w, X=FAKE, ws_bytes=1 << 40, saved=FAKE):
    return _lib.forward(sh, w, X, FAKE, FAKE, FAKE, saved, FAKE, ws_bytes, None)


def test_forward_argument_errors(L):
    sh = shape()
    assert fwd(L, sh, weights(Wg=None)) == _lib.ERR_INVALID_ARG
    assert fwd(L, sh, weights(Bd=FAKE + 2)) == _lib.ERR_MISALIGNED
    assert fwd(L, sh, weights(), X=None) == _lib.ERR_INVALID_ARG
    assert fwd(L, sh, weights(), X=FAKE + 8) == _lib.ERR_MISALIGNED
    assert fwd(L, sh, weights(), saved=None) == _lib.ERR_INVALID_ARG
    fws, _, _ = _lib.sizes(sh)
    assert fwd(L, sh, weights(), ws_bytes=fws - 1) == _lib.ERR_WORKSPACE_TOO_SMALL
    # int4 needs the scale pointers
    sh4 = shape(d_ff=768, fmt=1)
    assert fwd(L, sh4, weights()) == _lib.ERR_INVALID_ARG
    assert L.lora_mlp_forward(None, ctypes.byref(weights()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, None) \
        == _lib.ERR_INVALID_ARG


def test_backward_argument_errors(L):
    sh = shape()
    _, bws, _ = _lib.sizes(sh)
    g = _lib.Grads(*([FAKE] * 6))
    w = weights()

    def bwd(dOut=FAKE, grads=g, ws=bws):
        return _lib.backward(sh, w, FAKE, FAKE, FAKE, FAKE, dOut, FAKE, grads, FAKE, ws, None)

    assert bwd(dOut=None) == _lib.ERR_INVALID_ARG
    assert bwd(dOut=FAKE + 4) == _lib.ERR_MISALIGNED
    assert bwd(grads=_lib.Grads(FAKE, FAKE, None, FAKE, FAKE, FAKE)) == _lib.ERR_INVALID_ARG
    assert bwd(ws=bws - 1) == _lib.ERR_WORKSPACE_TOO_SMALL
    assert L.lora_mlp_backward(ctypes.byref(sh), ctypes.byref(w), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                               bws, None) == _lib.ERR_INVALID_ARG


def test_pointer_check_without_gpu(L):
    assert _lib.check_pointer(None) == _lib.ERR_INVALID_ARG
    assert _lib.check_pointer(FAKE + 8, 16) == _lib.ERR_MISALIGNED
    # an aligned address that no CUDA device owns (none here) is refused
    assert _lib.check_pointer(FAKE, 16) == _lib.ERR_INVALID_ARG


def test_dequant_argument_errors(L):
    assert _lib.dequant_int4(FAKE, FAKE, 4, 100, FAKE, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _lib.dequant_int4(FAKE, FAKE, 0, 64, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.dequant_int4(None, FAKE, 4, 64, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.dequant_int4(FAKE, FAKE + 1, 4, 64, FAKE, None) == _lib.ERR_MISALIGNED


def test_timing_toggle_without_gpu(L):
    _lib.timing_enable(True)
    _lib.timing_enable(False)
    assert _lib.timing_collect() == []
    assert _lib.launch_count() == 0


# ----------------------------------------------------------------------------- LoRA linear


def lshape(N=300, d_in=192, d_out=320, r=8, alpha=16.0, fmt=0):
    return _lib.make_lin_shape(N, d_in, d_out, r, alpha, fmt)


def test_linear_sizes(L):
    f1, b1, s1 = _lib.lin_sizes(lshape(N=300))
    f2, b2, s2 = _lib.lin_sizes(lshape(N=4096))
    assert 0 < f1 < f2 and 0 < b1 < b2 and 0 < s1 < s2
    assert s1 >= 8 * 304 * 2          # s X A^T kept as bf16 [r, N padded to 8]
    # int4 weights are dequantised inside the GEMMs: no bf16 copy in the scratch
    f4, b4, _ = _lib.lin_sizes(lshape(d_in=256, fmt=1))
    f0, b0, _ = _lib.lin_sizes(lshape(d_in=256, fmt=0))
    assert f4 - f0 < 320 * 256 * 2 // 16 and b4 - b0 < 320 * 256 * 2 // 16


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), _lib.ERR_INVALID_ARG),
    (dict(d_out=-8), _lib.ERR_INVALID_ARG),
    (dict(alpha=float("nan")), _lib.ERR_INVALID_ARG),
    (dict(fmt=3), _lib.ERR_INVALID_ARG),
    (dict(d_in=196), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(d_out=324), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(r=4), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(r=136), _lib.ERR_UNSUPPORTED_SHAPE),
    (dict(d_in=200, fmt=1), _lib.ERR_UNSUPPORTED_SHAPE),
])
def test_linear_shape_validation(L, kw, code):
    f = ctypes.c_size_t()
    assert L.lora_linear_sizes(ctypes.byref(lshape(**kw)), ctypes.byref(f), None, None) == code


def test_linear_argument_errors(L):
    sh = lshape()
    fws, bws, _ = _lib.lin_sizes(sh)
    w = _lib.LinWeights(FAKE, None, FAKE, FAKE)
    assert _lib.lin_forward(sh, w, FAKE, FAKE, FAKE, FAKE, fws - 1, None) == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.lin_forward(sh, w, None, FAKE, FAKE, FAKE, fws, None) == _lib.ERR_INVALID_ARG
    assert _lib.lin_forward(sh, _lib.LinWeights(FAKE, None, FAKE + 2, FAKE), FAKE, FAKE, FAKE, FAKE, fws,
                            None) == _lib.ERR_MISALIGNED
    assert _lib.lin_forward(lshape(d_in=256, fmt=1), w, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) \
        == _lib.ERR_INVALID_ARG     # int4 needs the scales
    assert _lib.lin_backward(sh, w, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, bws, None) == _lib.ERR_INVALID_ARG
    assert _lib.lin_backward(sh, w, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, FAKE, bws, None) \
        == _lib.ERR_MISALIGNED
    assert _lib.lin_backward(sh, w, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bws - 1, None) \
        == _lib.ERR_WORKSPACE_TOO_SMALL


# ----------------------------------------------------------------------------- RMSNorm and the block


def test_block_sizes_add_the_norm_buffers(L):
    sh = shape()
    f, b, s = _lib.sizes(sh)
    bf, bb, bs = _lib.block_sizes(sh)
    assert bf >= f + 512 * 256 * 2          # the normalised rows
    assert bb >= b + 2 * 512 * 256 * 2      # normalised rows and their gradient
    assert bs >= s + 512 * 4                # rstd


def test_norm_and_block_argument_errors(L):
    assert _lib.rmsnorm_forward(0, 64, 1e-5, FAKE, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.rmsnorm_forward(4, 60, 1e-5, FAKE, FAKE, FAKE, FAKE, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _lib.rmsnorm_forward(4, 64, -1.0, FAKE, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.rmsnorm_forward(4, 64, float("nan"), FAKE, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.rmsnorm_forward(4, 64, 1e-5, FAKE, None, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.rmsnorm_backward(4, 64, FAKE, FAKE, FAKE + 4, FAKE, FAKE, None) == _lib.ERR_MISALIGNED
    sh = shape()
    bf, bb, _ = _lib.block_sizes(sh)
    assert _lib.block_forward(sh, weights(), FAKE, 1e-5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bf - 1, None) \
        == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.block_forward(sh, weights(), None, 1e-5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bf, None) \
        == _lib.ERR_INVALID_ARG
    g = _lib.Grads(*([FAKE] * 6))
    assert _lib.block_backward(sh, weights(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, g, FAKE, bb - 1, None) \
        == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.block_backward(sh, weights(), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, g, FAKE, bb, None) \
        == _lib.ERR_INVALID_ARG


def test_folded_block_argument_errors(L):
    """The gamma-folded block takes bf16 frozen weights only, and the same
    workspace and saved sizes as the unfused block."""
    sh = shape()
    bf, bb, _ = _lib.block_sizes(sh)
    f, b, _ = _lib.sizes(sh)
    assert bf >= f + 512 * 256 * 2 + 2 * 8 * 256 * 2     # normalised rows and the two A diag(gamma)
    assert bb >= b + 2 * 512 * 256 * 2 + 2 * 8 * 256 * 2
    assert _lib.block_fold_gamma(sh, weights(), None, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.block_fold_gamma(sh, weights(), FAKE, FAKE + 8, FAKE, None) == _lib.ERR_MISALIGNED
    q = shape(d_ff=768, fmt=1)
    wq = weights(Sg=FAKE, Su=FAKE, Sd=FAKE)
    assert _lib.block_fold_gamma(q, wq, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert _lib.block_forward_folded(sh, weights(), FAKE, 1e-5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bf - 1, None) \
        == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.block_forward_folded(sh, weights(), None, 1e-5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bf, None) \
        == _lib.ERR_INVALID_ARG
    assert _lib.block_forward_folded(sh, weights(), FAKE, -1.0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, bf, None) \
        == _lib.ERR_INVALID_ARG
    qf, qb, _ = _lib.block_sizes(q)
    assert _lib.block_forward_folded(q, wq, FAKE, 1e-5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, qf, None) \
        == _lib.ERR_INVALID_ARG
    g = _lib.Grads(*([FAKE] * 6))
    assert _lib.block_backward_folded(sh, weights(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, g, FAKE, bb - 1,
                                      None) == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.block_backward_folded(sh, weights(), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, g, FAKE, bb, None) \
        == _lib.ERR_INVALID_ARG
    assert _lib.block_backward_folded(q, wq, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, g, FAKE, qb, None) \
        == _lib.ERR_INVALID_ARG


# ----------------------------------------------------------------------------- cross-entropy


def test_ce_sizes(L):
    ws = _lib.ce_sizes(_lib.make_ce_shape(4096, 256000))
    # one (max, sum) float2 per (row, 65536-logit chunk) and one float per row
    assert ws >= 4096 * 4 * 8 + 4096 * 4
    assert _lib.ce_sizes(_lib.make_ce_shape(1, 1, 8)) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), _lib.ERR_INVALID_ARG),
    (dict(V=0), _lib.ERR_INVALID_ARG),
    (dict(ld=999), _lib.ERR_INVALID_ARG),            # ld < V
    (dict(ld=1004), _lib.ERR_UNSUPPORTED_SHAPE),     # not a multiple of 8
    (dict(logit_scale=0.0), _lib.ERR_INVALID_ARG),
    (dict(logit_scale=float("nan")), _lib.ERR_INVALID_ARG),
    (dict(softcap=-1.0), _lib.ERR_INVALID_ARG),
    (dict(softcap=float("inf")), _lib.ERR_INVALID_ARG),
])
def test_ce_shape_validation(L, kw, code):
    args = dict(N=37, V=1000, ld=1000, logit_scale=1.0, softcap=0.0)
    args.update(kw)
    sh = _lib.make_ce_shape(**args)
    ws = ctypes.c_size_t()
    assert L.lora_ce_sizes(ctypes.byref(sh), ctypes.byref(ws)) == code


def test_ce_argument_errors(L):
    sh = _lib.make_ce_shape(37, 1000, 1008, 1.0, 30.0)
    ws = _lib.ce_sizes(sh)
    assert _lib.ce_forward(sh, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, None) == _lib.ERR_WORKSPACE_TOO_SMALL
    assert _lib.ce_forward(sh, None, FAKE, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert _lib.ce_forward(sh, FAKE + 8, FAKE, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_MISALIGNED
    assert _lib.ce_forward(sh, FAKE, FAKE + 4, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_MISALIGNED
    assert _lib.ce_backward(sh, FAKE, FAKE, FAKE, FAKE, None, None) == _lib.ERR_INVALID_ARG
    assert _lib.ce_backward(sh, FAKE, FAKE, FAKE, FAKE, FAKE + 2, None) == _lib.ERR_MISALIGNED
    assert _lib.ce_backward(sh, FAKE, FAKE, FAKE + 1, FAKE, FAKE, None) == _lib.ERR_MISALIGNED
    assert L.lora_ce_forward(None, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert L.lora_ce_device_status(None, None) == _lib.ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(), dict(N=4096, d=4096, d_ff=14336, r=16), dict(N=1, d=136, r=24),
                                dict(d=256, d_ff=704, fmt=1)])
def test_workspace_size_is_the_sizes_pair(L, kw):
    sh = shape(**kw)
    f, b, _ = _lib.sizes(sh)
    assert _lib.workspace_size(sh) == (f, b)
    one = ctypes.c_size_t()
    assert L.lora_mlp_workspace_size(ctypes.byref(sh), ctypes.byref(one), None) == _lib.OK and one.value == f
    bad = shape(d=250)
    assert (L.lora_mlp_workspace_size(ctypes.byref(bad), None, None)
            == L.lora_mlp_sizes(ctypes.byref(bad), None, None, None) == _lib.ERR_UNSUPPORTED_SHAPE)


def test_ce_reduced_argument_errors(L):
    sh = _lib.make_ce_shape(37, 1000, 1008, 1.0, 30.0)
    ws = _lib.ce_sizes(sh)
    mean = _lib.CE_REDUCTION_MEAN
    fr = _lib.ce_forward_reduced
    assert fr(sh, FAKE, FAKE, mean, FAKE, FAKE, FAKE, ws - 1, None) == _lib.ERR_WORKSPACE_TOO_SMALL
    assert fr(sh, FAKE, FAKE, 0, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG      # no reduction
    assert fr(sh, FAKE, FAKE, 3, FAKE, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert fr(sh, FAKE, FAKE, mean, None, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert fr(sh, FAKE, FAKE, mean, FAKE + 4, FAKE, FAKE, ws, None) == _lib.ERR_MISALIGNED  # out is 8-byte aligned
    br = _lib.ce_backward_reduced
    assert br(sh, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == _lib.ERR_INVALID_ARG
    assert br(sh, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, None) == _lib.ERR_MISALIGNED
    assert br(sh, FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, None) == _lib.ERR_MISALIGNED
