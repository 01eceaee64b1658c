"""PyTorch-facing wrappers of the C ABI.

PyTorch provides device memory and the current stream; every step of the
LoRA SwiGLU MLP and of the LoRA linear runs in the library's sm_100a kernels.  There is no fallback:
if the CUDA library is missing or the device is not a B200 the call raises.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib

BF16 = torch.bfloat16


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


@dataclass
class MLPWeights:
    """Frozen SwiGLU weights and the three LoRA adapters (nn.Linear layout).

    bf16 weights: Wg, Wu [d_ff, d], Wd [d, d_ff].  int4 weights: Wg, Wu uint8
    [d_ff, d/2], Wd uint8 [d, d_ff/2] and fp16 scales Sg, Su [d_ff, d/64],
    Sd [d, d_ff/64].  FP8 weights: Wg, Wu float8_e4m3fn [d_ff, d], Wd
    float8_e4m3fn [d, d_ff] and fp32 scales of the int4 shapes.  Adapters (bf16): Ag, Au [r, d]; Bg, Bu [d_ff, r];
    Ad [r, d_ff]; Bd [d, r].
    """
    Wg: torch.Tensor
    Wu: torch.Tensor
    Wd: torch.Tensor
    Ag: torch.Tensor
    Bg: torch.Tensor
    Au: torch.Tensor
    Bu: torch.Tensor
    Ad: torch.Tensor
    Bd: torch.Tensor
    alpha: float
    Sg: torch.Tensor | None = None
    Su: torch.Tensor | None = None
    Sd: torch.Tensor | None = None

    @property
    def int4(self) -> bool:
        return self.Wg.dtype == torch.uint8

    @property
    def fp8(self) -> bool:
        return self.Wg.dtype == torch.float8_e4m3fn

    @property
    def fmt(self) -> int:
        return _lib.WEIGHTS_INT4_B64 if self.int4 else (_lib.WEIGHTS_FP8_B64 if self.fp8 else _lib.WEIGHTS_BF16)

    @property
    def r(self) -> int:
        return int(self.Ag.shape[0])

    @property
    def d(self) -> int:
        return int(self.Ag.shape[1])

    @property
    def d_ff(self) -> int:
        return int(self.Bg.shape[0])

    def shape(self, N: int) -> _lib.Shape:
        return _lib.make_shape(N, self.d, self.d_ff, self.r, self.alpha, self.fmt)

    def validate(self):
        d, d_ff, r = self.d, self.d_ff, self.r
        if self.int4:
            _need(self.Wg, "Wg", torch.uint8, (d_ff, d // 2))
            _need(self.Wu, "Wu", torch.uint8, (d_ff, d // 2))
            _need(self.Wd, "Wd", torch.uint8, (d, d_ff // 2))
            _need(self.Sg, "Sg", torch.float16, (d_ff, d // 64))
            _need(self.Su, "Su", torch.float16, (d_ff, d // 64))
            _need(self.Sd, "Sd", torch.float16, (d, d_ff // 64))
        elif self.fp8:
            _need(self.Wg, "Wg", torch.float8_e4m3fn, (d_ff, d))
            _need(self.Wu, "Wu", torch.float8_e4m3fn, (d_ff, d))
            _need(self.Wd, "Wd", torch.float8_e4m3fn, (d, d_ff))
            _need(self.Sg, "Sg", torch.float32, (d_ff, d // 64))
            _need(self.Su, "Su", torch.float32, (d_ff, d // 64))
            _need(self.Sd, "Sd", torch.float32, (d, d_ff // 64))
        else:
            _need(self.Wg, "Wg", BF16, (d_ff, d))
            _need(self.Wu, "Wu", BF16, (d_ff, d))
            _need(self.Wd, "Wd", BF16, (d, d_ff))
        _need(self.Ag, "Ag", BF16, (r, d))
        _need(self.Au, "Au", BF16, (r, d))
        _need(self.Bg, "Bg", BF16, (d_ff, r))
        _need(self.Bu, "Bu", BF16, (d_ff, r))
        _need(self.Ad, "Ad", BF16, (r, d_ff))
        _need(self.Bd, "Bd", BF16, (d, r))

    def c_struct(self) -> _lib.Weights:
        return _lib.Weights(*[None if getattr(self, n) is None else getattr(self, n).data_ptr()
                              for n in _lib.WEIGHT_FIELDS])


@dataclass
class Saved:
    """What forward keeps for backward: the bf16 pre-activations g, u and the
    library's opaque rank-r buffer."""
    g: torch.Tensor
    u: torch.Tensor
    lowrank: torch.Tensor


class Workspace:
    """A reusable device scratch buffer (grown on demand)."""

    def __init__(self):
        self.buf = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


def sizes(w: MLPWeights, N: int):
    """(forward workspace, backward workspace, saved) byte counts."""
    return _lib.sizes(w.shape(N))


def forward(X: torch.Tensor, w: MLPWeights, *, out=None, workspace: Workspace | None = None, stream=None):
    """out = MLP(X).  Returns (out, Saved)."""
    N, d = X.shape
    _need(X, "X", BF16, (N, w.d))
    w.validate()
    shape = w.shape(N)
    fws, _, svs = _lib.sizes(shape)
    dev = X.device
    out = torch.empty((N, d), dtype=BF16, device=dev) if out is None else _need(out, "out", BF16, (N, d))
    g = torch.empty((N, w.d_ff), dtype=BF16, device=dev)
    u = torch.empty((N, w.d_ff), dtype=BF16, device=dev)
    lowrank = torch.empty(max(svs, 256), dtype=torch.uint8, device=dev)
    ws = (workspace or Workspace()).get(fws, dev)
    _lib.check(_lib.forward(shape, w.c_struct(), _p(X), _p(out), _p(g), _p(u), _p(lowrank), _p(ws),
                            ws.numel(), _stream(stream)), "lora_mlp_forward")
    return out, Saved(g, u, lowrank)


def backward(X: torch.Tensor, w: MLPWeights, saved: Saved, dOut: torch.Tensor, *, dX=None, grads=None,
             workspace: Workspace | None = None, stream=None):
    """Returns (dX, {dAg, dBg, dAu, dBu, dAd, dBd})."""
    N, d = X.shape
    _need(X, "X", BF16, (N, w.d))
    _need(dOut, "dOut", BF16, (N, d))
    w.validate()
    shape = w.shape(N)
    _, bws, _ = _lib.sizes(shape)
    dev = X.device
    dX = torch.empty((N, d), dtype=BF16, device=dev) if dX is None else _need(dX, "dX", BF16, (N, d))
    if grads is None:
        grads = {("d" + k): torch.empty_like(getattr(w, k)) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    gs = _lib.Grads(*[grads[k].data_ptr() for k in _lib.GRAD_FIELDS])
    ws = (workspace or Workspace()).get(bws, dev)
    _lib.check(_lib.backward(shape, w.c_struct(), _p(X), _p(saved.g), _p(saved.u), _p(saved.lowrank), _p(dOut),
                             _p(dX), gs, _p(ws), ws.numel(), _stream(stream)), "lora_mlp_backward")
    return dX, grads


def dequant_int4(packed: torch.Tensor, scales: torch.Tensor, stream=None) -> torch.Tensor:
    rows, half = packed.shape
    _need(packed, "packed", torch.uint8)
    _need(scales, "scales", torch.float16, (rows, 2 * half // 64))
    w = torch.empty((rows, 2 * half), dtype=BF16, device=packed.device)
    _lib.check(_lib.dequant_int4(_p(packed), _p(scales), rows, 2 * half, _p(w), _stream(stream)),
               "lora_mlp_dequant_int4")
    return w


def dequant_fp8(codes: torch.Tensor, scales: torch.Tensor, stream=None) -> torch.Tensor:
    """bf16 [rows, cols] from FP8 E4M3 codes [rows, cols] (float8_e4m3fn or
    uint8) and fp32 block scales [rows, cols/64], by the library's kernel."""
    rows, cols = codes.shape
    if codes.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError("codes must be float8_e4m3fn or uint8")
    _need(scales, "scales", torch.float32, (rows, cols // 64))
    w = torch.empty((rows, cols), dtype=BF16, device=codes.device)
    _lib.check(_lib.dequant_fp8(_p(codes), _p(scales), rows, cols, _p(w), _stream(stream)), "lora_mlp_dequant_fp8")
    return w


class LoRAMLPFunction(torch.autograd.Function):
    """autograd wrapper: out = LoRA-SwiGLU-MLP(X); backward fills X.grad and the
    adapter grads.  Usage: LoRAMLPFunction.apply(X, w, Ag, Bg, Au, Bu, Ad, Bd)
    where w is an MLPWeights whose adapter tensors are the same objects."""

    @staticmethod
    def forward(ctx, X, w: MLPWeights, Ag, Bg, Au, Bu, Ad, Bd):
        out, saved = forward(X.contiguous(), w)
        ctx.w = w
        ctx.saved_lr = saved
        ctx.save_for_backward(X)
        return out

    @staticmethod
    def backward(ctx, dOut):
        (X,) = ctx.saved_tensors
        dX, g = backward(X, ctx.w, ctx.saved_lr, dOut.contiguous())
        return dX, None, g["dAg"], g["dBg"], g["dAu"], g["dBu"], g["dAd"], g["dBd"]


def weights_from_host(inp: dict, alpha: float, device="cuda") -> MLPWeights:
    """Upload a host input dict (bf16 bits as uint16 numpy arrays, int4 as
    packed uint8 + fp16 scales) to the device."""
    def bf(a):
        return torch.from_numpy(a.view("int16")).view(BF16).to(device)

    kw = {}
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        kw[k] = bf(inp[k])
    if "Wg_q" in inp:
        for k, s in (("Wg", "Sg"), ("Wu", "Su"), ("Wd", "Sd")):
            kw[k] = torch.from_numpy(inp[k + "_q"]).to(device)
            kw[s] = torch.from_numpy(inp[k + "_scale"]).to(device)
    elif "Wg_f8" in inp:
        for k, s in (("Wg", "Sg"), ("Wu", "Su"), ("Wd", "Sd")):
            kw[k] = torch.from_numpy(inp[k + "_f8"]).view(torch.float8_e4m3fn).to(device)
            kw[s] = torch.from_numpy(inp[k + "_f8scale"]).to(device)
    else:
        for k in ("Wg", "Wu", "Wd"):
            kw[k] = bf(inp[k])
    return MLPWeights(alpha=float(alpha), **kw)


def to_device_bf16(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(a.view("int16")).view(BF16).to(device)


class HostBatchTrainer:
    """Forward + backward over batches that live in (pinned) host memory.

    The host-to-device copy of the next batch runs on its own stream while the
    current batch computes, and each step's adapter gradients are copied back
    to pinned host memory on a third stream while the next step computes.
    Inputs and gradients are double-buffered on the device (and the
    gradients on the host), ordered by CUDA events: a device buffer is
    refilled only once the step that used it, or its copy back, is done.
    Every step still moves its own inputs and result across PCIe; only the
    overlap with compute is new.
    """

    def __init__(self, w: MLPWeights, N: int, device=None, gamma: torch.Tensor | None = None, eps: float = 1e-5):
        """With `gamma`, each step runs the pre-norm block MLP(RMSNorm(X))."""
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.w, self.N, self.dev = w, N, dev
        self.gamma, self.eps = gamma, eps
        d = w.d
        self.X = [torch.empty((N, d), dtype=BF16, device=dev) for _ in range(2)]
        self.dOut = [torch.empty((N, d), dtype=BF16, device=dev) for _ in range(2)]
        self.out = torch.empty((N, d), dtype=BF16, device=dev)
        self.dX = torch.empty((N, d), dtype=BF16, device=dev)
        names = ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")
        self.grads = [{("d" + k): torch.empty_like(getattr(w, k)) for k in names} for _ in range(2)]
        self.grads_host = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in g.items()}
                           for g in self.grads]
        self.wsf, self.wsb = Workspace(), Workspace()
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.d2h_stream = torch.cuda.Stream(device=dev)
        self.ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.free = [torch.cuda.Event(), torch.cuda.Event()]
        self.computed = [torch.cuda.Event(), torch.cuda.Event()]
        self.fetched = [torch.cuda.Event(), torch.cuda.Event()]
        self.fetch_pending = [False, False]
        self.slot = 0
        self.primed = False

    def _stage(self, slot, Xh, dOh):
        with torch.cuda.stream(self.copy_stream):
            self.copy_stream.wait_event(self.free[slot])
            self.X[slot].copy_(Xh, non_blocking=True)
            self.dOut[slot].copy_(dOh, non_blocking=True)
            self.ready[slot].record(self.copy_stream)

    def h2d_bytes(self) -> int:
        return 2 * self.N * self.w.d * 2

    def d2h_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.grads[0].values())

    def step(self, Xh, dOh, next_Xh=None, next_dOh=None):
        """One training step on host batch (Xh, dOh); if the next batch is
        given, its copy is started so that it overlaps this step's compute.
        Returns the dict of pinned host adapter gradients of this step: valid
        after `finish()` and a synchronisation of the current stream (or the
        device), and until the step after next overwrites them."""
        cur = self.slot
        if not self.primed:
            self._stage(cur, Xh, dOh)
            self.primed = True
        nxt = cur ^ 1
        if next_Xh is not None:
            self._stage(nxt, next_Xh, next_dOh)
        stream = torch.cuda.current_stream(self.dev)
        stream.wait_event(self.ready[cur])
        if self.fetch_pending[cur]:
            stream.wait_event(self.fetched[cur])  # this slot's gradients from two steps ago are home
        grads = self.grads[cur]
        if self.gamma is None:
            o, saved = forward(self.X[cur], self.w, out=self.out, workspace=self.wsf)
            backward(self.X[cur], self.w, saved, self.dOut[cur], dX=self.dX, grads=grads, workspace=self.wsb)
        else:
            o, saved = block_forward(self.X[cur], self.w, self.gamma, self.eps, out=self.out, workspace=self.wsf)
            block_backward(self.X[cur], self.w, self.gamma, saved, self.dOut[cur], dX=self.dX, grads=grads,
                           workspace=self.wsb)
        self.free[cur].record(stream)
        self.computed[cur].record(stream)
        with torch.cuda.stream(self.d2h_stream):
            self.d2h_stream.wait_event(self.computed[cur])
            for k, v in grads.items():
                self.grads_host[cur][k].copy_(v, non_blocking=True)
            self.fetched[cur].record(self.d2h_stream)
        self.fetch_pending[cur] = True
        self.slot = nxt
        if next_Xh is None:
            self.primed = False
        return self.grads_host[cur]

    def finish(self):
        """Orders the current stream after every gradient copy issued so far."""
        stream = torch.cuda.current_stream(self.dev)
        for i in range(2):
            if self.fetch_pending[i]:
                stream.wait_event(self.fetched[i])


# ----------------------------------------------------------------------------- LoRA linear


@dataclass
class LinearWeights:
    """One frozen projection with a LoRA adapter (nn.Linear layout).

    bf16: W [d_out, d_in].  int4: W uint8 [d_out, d_in/2] and fp16 scales
    S [d_out, d_in/64].  FP8: W float8_e4m3fn [d_out, d_in] and fp32 scales
    S [d_out, d_in/64].  Adapter (bf16): A [r, d_in], B [d_out, r].
    """
    W: torch.Tensor
    A: torch.Tensor
    B: torch.Tensor
    alpha: float
    S: torch.Tensor | None = None

    @property
    def int4(self) -> bool:
        return self.W.dtype == torch.uint8

    @property
    def fp8(self) -> bool:
        return self.W.dtype == torch.float8_e4m3fn

    @property
    def r(self) -> int:
        return int(self.A.shape[0])

    @property
    def d_in(self) -> int:
        return int(self.A.shape[1])

    @property
    def d_out(self) -> int:
        return int(self.B.shape[0])

    def shape(self, N: int) -> _lib.LinShape:
        fmt = _lib.WEIGHTS_INT4_B64 if self.int4 else (_lib.WEIGHTS_FP8_B64 if self.fp8 else _lib.WEIGHTS_BF16)
        return _lib.make_lin_shape(N, self.d_in, self.d_out, self.r, self.alpha, fmt)

    def validate(self):
        di, do, r = self.d_in, self.d_out, self.r
        if self.int4:
            _need(self.W, "W", torch.uint8, (do, di // 2))
            _need(self.S, "S", torch.float16, (do, di // 64))
        elif self.fp8:
            _need(self.W, "W", torch.float8_e4m3fn, (do, di))
            _need(self.S, "S", torch.float32, (do, di // 64))
        else:
            _need(self.W, "W", BF16, (do, di))
        _need(self.A, "A", BF16, (r, di))
        _need(self.B, "B", BF16, (do, r))

    def c_struct(self) -> _lib.LinWeights:
        return _lib.LinWeights(self.W.data_ptr(), None if self.S is None else self.S.data_ptr(),
                               self.A.data_ptr(), self.B.data_ptr())


def linear_sizes(w: LinearWeights, N: int):
    """(forward workspace, backward workspace, saved) byte counts."""
    return _lib.lin_sizes(w.shape(N))


def linear_forward(X: torch.Tensor, w: LinearWeights, *, Y=None, workspace: Workspace | None = None,
                   stream=None):
    """Y = X (W + s B A)^T.  Returns (Y, saved) where saved is the opaque
    rank-r buffer backward needs."""
    N = X.shape[0]
    _need(X, "X", BF16, (N, w.d_in))
    w.validate()
    shape = w.shape(N)
    fws, _, svs = _lib.lin_sizes(shape)
    dev = X.device
    Y = torch.empty((N, w.d_out), dtype=BF16, device=dev) if Y is None else _need(Y, "Y", BF16, (N, w.d_out))
    saved = torch.empty(max(svs, 256), dtype=torch.uint8, device=dev)
    ws = (workspace or Workspace()).get(fws, dev)
    _lib.check(_lib.lin_forward(shape, w.c_struct(), _p(X), _p(Y), _p(saved), _p(ws), ws.numel(),
                                _stream(stream)), "lora_linear_forward")
    return Y, saved


def linear_backward(X: torch.Tensor, w: LinearWeights, saved: torch.Tensor, dY: torch.Tensor, *, dX=None,
                    dA=None, dB=None, workspace: Workspace | None = None, stream=None):
    """Returns (dX, dA, dB)."""
    N = X.shape[0]
    _need(X, "X", BF16, (N, w.d_in))
    _need(dY, "dY", BF16, (N, w.d_out))
    w.validate()
    shape = w.shape(N)
    _, bws, _ = _lib.lin_sizes(shape)
    dev = X.device
    dX = torch.empty((N, w.d_in), dtype=BF16, device=dev) if dX is None else _need(dX, "dX", BF16, (N, w.d_in))
    dA = torch.empty_like(w.A) if dA is None else _need(dA, "dA", BF16, tuple(w.A.shape))
    dB = torch.empty_like(w.B) if dB is None else _need(dB, "dB", BF16, tuple(w.B.shape))
    ws = (workspace or Workspace()).get(bws, dev)
    _lib.check(_lib.lin_backward(shape, w.c_struct(), _p(X), _p(saved), _p(dY), _p(dX), _p(dA), _p(dB), _p(ws),
                                 ws.numel(), _stream(stream)), "lora_linear_backward")
    return dX, dA, dB


class LoRALinearFunction(torch.autograd.Function):
    """autograd wrapper: Y = X (W + s B A)^T.  Usage:
    LoRALinearFunction.apply(X, w, A, B) where w is a LinearWeights whose A and
    B are the same tensors."""

    @staticmethod
    def forward(ctx, X, w: LinearWeights, A, B):
        Y, saved = linear_forward(X.contiguous(), w)
        ctx.w = w
        ctx.saved_lr = saved
        ctx.save_for_backward(X)
        return Y

    @staticmethod
    def backward(ctx, dY):
        (X,) = ctx.saved_tensors
        dX, dA, dB = linear_backward(X, ctx.w, ctx.saved_lr, dY.contiguous())
        return dX, None, dA, dB


def linear_weights_from_host(inp: dict, alpha: float, device="cuda") -> LinearWeights:
    """Upload a host LoRA-linear input dict to the device."""
    if "W_q" in inp:
        return LinearWeights(W=torch.from_numpy(inp["W_q"]).to(device), A=to_device_bf16(inp["A"], device),
                             B=to_device_bf16(inp["B"], device), alpha=float(alpha),
                             S=torch.from_numpy(inp["W_scale"]).to(device))
    if "W_f8" in inp:
        return LinearWeights(W=torch.from_numpy(inp["W_f8"]).view(torch.float8_e4m3fn).to(device),
                             A=to_device_bf16(inp["A"], device), B=to_device_bf16(inp["B"], device),
                             alpha=float(alpha), S=torch.from_numpy(inp["W_f8scale"]).to(device))
    return LinearWeights(W=to_device_bf16(inp["W"], device), A=to_device_bf16(inp["A"], device),
                         B=to_device_bf16(inp["B"], device), alpha=float(alpha))


# ----------------------------------------------------------------------------- RMSNorm and the pre-norm block


def rmsnorm_forward(x: torch.Tensor, gamma: torch.Tensor, eps: float, *, stream=None):
    """Returns (y, rstd): y = RMSNorm(x) * gamma (bf16), rstd fp32 [N]."""
    N, d = x.shape
    _need(x, "x", BF16)
    _need(gamma, "gamma", BF16, (d,))
    y = torch.empty_like(x)
    rstd = torch.empty((N,), dtype=torch.float32, device=x.device)
    _lib.check(_lib.rmsnorm_forward(N, d, eps, _p(x), _p(gamma), _p(y), _p(rstd), _stream(stream)),
               "lora_rmsnorm_forward")
    return y, rstd


def rmsnorm_backward(x: torch.Tensor, gamma: torch.Tensor, rstd: torch.Tensor, dy: torch.Tensor, *, stream=None):
    N, d = x.shape
    _need(x, "x", BF16)
    _need(gamma, "gamma", BF16, (d,))
    _need(rstd, "rstd", torch.float32, (N,))
    _need(dy, "dy", BF16, (N, d))
    dx = torch.empty_like(x)
    _lib.check(_lib.rmsnorm_backward(N, d, _p(x), _p(gamma), _p(rstd), _p(dy), _p(dx), _stream(stream)),
               "lora_rmsnorm_backward")
    return dx


class RMSNormFunction(torch.autograd.Function):
    """autograd wrapper of the library's RMSNorm: y = x * rstd * gamma per row,
    with the frozen gain gamma (no gradient for it) and the forward's rstd
    reused by the backward.  Usage: RMSNormFunction.apply(x, gamma, eps)."""

    @staticmethod
    def forward(ctx, x, gamma, eps=1e-5):
        x = x.contiguous()
        y, rstd = rmsnorm_forward(x, gamma, eps)
        ctx.save_for_backward(x, gamma, rstd)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, gamma, rstd = ctx.saved_tensors
        return rmsnorm_backward(x, gamma, rstd, dy.contiguous()), None, None


def fold_gamma(w: MLPWeights, gamma: torch.Tensor, stream=None) -> MLPWeights:
    """The weights of the fused-norm block: Wg, Wu with gamma folded into
    their columns (bf16_rne(W * gamma), by the library's kernel); Wd and the
    adapters are the same tensors as w's.  bf16 frozen weights only.  Done
    once: W and gamma are frozen."""
    if w.int4 or w.fp8:
        raise ValueError("gamma folds into bf16 frozen weights only")
    w.validate()
    _need(gamma, "gamma", BF16, (w.d,))
    Wg, Wu = torch.empty_like(w.Wg), torch.empty_like(w.Wu)
    _lib.check(_lib.block_fold_gamma(w.shape(1), w.c_struct(), _p(gamma), _p(Wg), _p(Wu), _stream(stream)),
               "lora_mlp_block_fold_gamma")
    return MLPWeights(Wg=Wg, Wu=Wu, Wd=w.Wd, Ag=w.Ag, Bg=w.Bg, Au=w.Au, Bu=w.Bu, Ad=w.Ad, Bd=w.Bd, alpha=w.alpha)


def block_forward(X: torch.Tensor, w: MLPWeights, gamma: torch.Tensor, eps: float, *, out=None,
                  workspace: Workspace | None = None, stream=None, folded: bool = False):
    """out = MLP(RMSNorm(X) * gamma).  Returns (out, Saved); Saved.lowrank
    also holds the per-row rstd.  folded=True: w comes from fold_gamma and
    the norm runs fused into the gate/up GEMM (lora_mlp_block_forward_folded)."""
    N, d = X.shape
    _need(X, "X", BF16, (N, w.d))
    _need(gamma, "gamma", BF16, (w.d,))
    w.validate()
    shape = w.shape(N)
    fws, _, svs = _lib.block_sizes(shape)
    dev = X.device
    out = torch.empty((N, d), dtype=BF16, device=dev) if out is None else _need(out, "out", BF16, (N, d))
    g = torch.empty((N, w.d_ff), dtype=BF16, device=dev)
    u = torch.empty((N, w.d_ff), dtype=BF16, device=dev)
    saved = torch.empty(max(svs, 256), dtype=torch.uint8, device=dev)
    ws = (workspace or Workspace()).get(fws, dev)
    fn = _lib.block_forward_folded if folded else _lib.block_forward
    _lib.check(fn(shape, w.c_struct(), _p(gamma), eps, _p(X), _p(out), _p(g), _p(u), _p(saved), _p(ws), ws.numel(),
                  _stream(stream)), "lora_mlp_block_forward" + ("_folded" if folded else ""))
    return out, Saved(g, u, saved)


def block_backward(X: torch.Tensor, w: MLPWeights, gamma: torch.Tensor, saved: Saved, dOut: torch.Tensor, *,
                   dX=None, grads=None, workspace: Workspace | None = None, stream=None, folded: bool = False):
    """Returns (dX, {dAg, dBg, dAu, dBu, dAd, dBd}) for the block input X.
    folded as in block_forward (and the same as the forward's)."""
    N, d = X.shape
    _need(X, "X", BF16, (N, w.d))
    _need(gamma, "gamma", BF16, (w.d,))
    _need(dOut, "dOut", BF16, (N, d))
    w.validate()
    shape = w.shape(N)
    _, bws, _ = _lib.block_sizes(shape)
    dev = X.device
    dX = torch.empty((N, d), dtype=BF16, device=dev) if dX is None else _need(dX, "dX", BF16, (N, d))
    if grads is None:
        grads = {("d" + k): torch.empty_like(getattr(w, k)) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    gs = _lib.Grads(*[grads[k].data_ptr() for k in _lib.GRAD_FIELDS])
    ws = (workspace or Workspace()).get(bws, dev)
    fn = _lib.block_backward_folded if folded else _lib.block_backward
    _lib.check(fn(shape, w.c_struct(), _p(gamma), _p(X), _p(saved.g), _p(saved.u), _p(saved.lowrank), _p(dOut),
                  _p(dX), gs, _p(ws), ws.numel(), _stream(stream)),
               "lora_mlp_block_backward" + ("_folded" if folded else ""))
    return dX, grads


class LoRAMLPBlockFunction(torch.autograd.Function):
    """autograd wrapper of the pre-norm block: out = MLP(RMSNorm(X) * gamma).
    Usage: LoRAMLPBlockFunction.apply(X, w, gamma, eps, Ag, Bg, Au, Bu, Ad, Bd)
    (gamma frozen: no gradient)."""

    @staticmethod
    def forward(ctx, X, w: MLPWeights, gamma, eps, Ag, Bg, Au, Bu, Ad, Bd):
        out, saved = block_forward(X.contiguous(), w, gamma, eps)
        ctx.w, ctx.gamma, ctx.saved_lr = w, gamma, saved
        ctx.save_for_backward(X)
        return out

    @staticmethod
    def backward(ctx, dOut):
        (X,) = ctx.saved_tensors
        dX, g = block_backward(X, ctx.w, ctx.gamma, ctx.saved_lr, dOut.contiguous())
        return dX, None, None, None, g["dAg"], g["dBg"], g["dAu"], g["dBu"], g["dAd"], g["dBd"]


# ----------------------------------------------------------------------------- chunked cross-entropy


def _ce_shape(logits: torch.Tensor, logit_scale: float, softcap: float, ignore_index: int):
    if logits.dim() != 2:
        raise ValueError("logits must be [N, V]")
    if logits.dtype != BF16 or not logits.is_cuda:
        raise TypeError("logits must be a bf16 CUDA tensor")
    if logits.stride(1) != 1:
        raise ValueError("logits rows must be contiguous")
    N, V = logits.shape
    return _lib.make_ce_shape(N, V, logits.stride(0), logit_scale, softcap, ignore_index)


def ce_forward(logits: torch.Tensor, labels: torch.Tensor, *, logit_scale: float = 1.0, softcap: float = 0.0,
               ignore_index: int = -100, workspace: Workspace | None = None, stream=None):
    """Per-row cross-entropy of bf16 logits [N, V] (row stride a multiple of
    8) against int64 labels [N]: returns (loss [N] fp32, lse [N] fp32), loss 0
    for rows labelled ignore_index."""
    shape = _ce_shape(logits, logit_scale, softcap, ignore_index)
    N = shape.N
    _need(labels, "labels", torch.int64, (N,))
    dev = logits.device
    loss = torch.empty((N,), dtype=torch.float32, device=dev)
    lse = torch.empty((N,), dtype=torch.float32, device=dev)
    ws = (workspace or Workspace()).get(_lib.ce_sizes(shape), dev)
    _lib.check(_lib.ce_forward(shape, _p(logits), _p(labels), _p(loss), _p(lse), _p(ws), ws.numel(),
                               _stream(stream)), "lora_ce_forward")
    return loss, lse


def ce_backward(logits: torch.Tensor, labels: torch.Tensor, lse: torch.Tensor, dloss: torch.Tensor, *,
                logit_scale: float = 1.0, softcap: float = 0.0, ignore_index: int = -100, out=None,
                inplace: bool = False, stream=None):
    """dlogits [N, V] bf16 for the per-row upstream gradient dloss [N] (fp32).
    inplace=True writes the gradient over the logits."""
    shape = _ce_shape(logits, logit_scale, softcap, ignore_index)
    N = shape.N
    _need(labels, "labels", torch.int64, (N,))
    _need(lse, "lse", torch.float32, (N,))
    _need(dloss, "dloss", torch.float32, (N,))
    # The kernel writes the gradient with the logits' row stride, so the
    # output keeps the logits' strides (empty_like would not for a padded view).
    if inplace:
        out = logits
    elif out is None:
        out = torch.empty_strided(logits.size(), logits.stride(), dtype=BF16, device=logits.device)
    elif (out.shape != logits.shape or out.stride() != logits.stride() or out.dtype != BF16 or not out.is_cuda):
        raise ValueError("out must have the logits' shape, strides and dtype")
    _lib.check(_lib.ce_backward(shape, _p(logits), _p(labels), _p(lse), _p(dloss), _p(out), _stream(stream)),
               "lora_ce_backward")
    return out


def ce_loss(logits: torch.Tensor, labels: torch.Tensor, *, reduction: str = "mean", logit_scale: float = 1.0,
            softcap: float = 0.0, ignore_index: int = -100, workspace: Workspace | None = None, stream=None):
    """The cross-entropy reduced over the rows, computed by the library:
    returns (out [2] fp32, lse [N] fp32), out[0] the summed or mean loss and
    out[1] its derivative with respect to each row's loss (1, or 1 / rows
    taking part), the factor ce_backward_reduced applies."""
    red = {"sum": _lib.CE_REDUCTION_SUM, "mean": _lib.CE_REDUCTION_MEAN}.get(reduction)
    if red is None:
        raise ValueError("reduction must be 'sum' or 'mean'")
    shape = _ce_shape(logits, logit_scale, softcap, ignore_index)
    N = shape.N
    _need(labels, "labels", torch.int64, (N,))
    dev = logits.device
    out = torch.empty((2,), dtype=torch.float32, device=dev)
    lse = torch.empty((N,), dtype=torch.float32, device=dev)
    ws = (workspace or Workspace()).get(_lib.ce_sizes(shape), dev)
    _lib.check(_lib.ce_forward_reduced(shape, _p(logits), _p(labels), red, _p(out), _p(lse), _p(ws), ws.numel(),
                                       _stream(stream)), "lora_ce_forward_reduced")
    return out, lse


def ce_backward_reduced(logits: torch.Tensor, labels: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                        fwd_out: torch.Tensor, *, logit_scale: float = 1.0, softcap: float = 0.0,
                        ignore_index: int = -100, out=None, inplace: bool = False, stream=None):
    """dlogits [N, V] bf16 for the upstream gradient dout (fp32, one element)
    of the loss ce_loss returned in fwd_out.  inplace=True writes the
    gradient over the logits."""
    shape = _ce_shape(logits, logit_scale, softcap, ignore_index)
    N = shape.N
    _need(labels, "labels", torch.int64, (N,))
    _need(lse, "lse", torch.float32, (N,))
    _need(fwd_out, "fwd_out", torch.float32, (2,))
    if dout.numel() != 1 or dout.dtype != torch.float32 or not dout.is_cuda:
        raise TypeError("dout must be one fp32 CUDA element")
    if inplace:
        out = logits
    elif out is None:
        out = torch.empty_strided(logits.size(), logits.stride(), dtype=BF16, device=logits.device)
    elif (out.shape != logits.shape or out.stride() != logits.stride() or out.dtype != BF16 or not out.is_cuda):
        raise ValueError("out must have the logits' shape, strides and dtype")
    _lib.check(_lib.ce_backward_reduced(shape, _p(logits), _p(labels), _p(lse), _p(dout), _p(fwd_out), _p(out),
                                        _stream(stream)), "lora_ce_backward_reduced")
    return out


class CrossEntropyFunction(torch.autograd.Function):
    """Mean cross-entropy over the rows whose label is not ignore_index, with
    the library's chunked kernels; the mean and its gradient factor are
    computed in the library.  Usage:
    CrossEntropyFunction.apply(logits, labels, logit_scale, softcap, ignore_index, inplace).
    By default the backward writes the logits' gradient to a new buffer.
    inplace=True writes it over the logits instead, as the pages' kernel does
    to save memory; the logits' version counter is then bumped, so any other
    autograd node that saved them raises instead of reading the gradient."""

    @staticmethod
    def forward(ctx, logits, labels, logit_scale=1.0, softcap=0.0, ignore_index=-100, inplace=False):
        out, lse = ce_loss(logits, labels, reduction="mean", logit_scale=logit_scale, softcap=softcap,
                           ignore_index=ignore_index)
        ctx.save_for_backward(logits, labels, lse, out)
        ctx.cfg = (logit_scale, softcap, ignore_index, bool(inplace))
        return out[0]

    @staticmethod
    def backward(ctx, g):
        logits, labels, lse, out = ctx.saved_tensors
        s, c, ign, inplace = ctx.cfg
        if g.dtype != torch.float32 or not g.is_cuda:
            raise TypeError("the upstream gradient of the loss must be fp32 on the GPU")
        dz = ce_backward_reduced(logits, labels, lse, g.contiguous(), out, logit_scale=s, softcap=c,
                                 ignore_index=ign, inplace=inplace)
        if inplace:
            torch.autograd.graph.increment_version(logits)
        return dz, None, None, None, None, None
