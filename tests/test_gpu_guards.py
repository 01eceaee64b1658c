"""Write coverage and overruns, through the C ABI.

Each output buffer is the front of a larger allocation: its body starts as
NaN (bf16 0xFFFF) and a guard zone after its end holds a canary byte.  The
workspaces start as NaN garbage too.  After forward + backward every output
element must have been written (no NaN left), every guard must be intact,
and the results must equal, bit for bit, a second run whose buffers and
workspaces started as zeros: no kernel reads memory it did not write first.
Ragged shapes put tile edges inside the buffers' last rows and columns."""
import ctypes

import pytest
import torch

from lora_fine_tuning_mlp_b200 import _lib, api
from lora_fine_tuning_mlp_b200 import build as libbuild
from lora_fine_tuning_mlp_b200 import inputs as synth

pytestmark = pytest.mark.gpu
GUARD = 4096
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


class Carved:
    """`nbytes` of body (filled with `body`) followed by a canary guard zone."""

    def __init__(self, nbytes: int, body: int, dev):
        self.nbytes = nbytes
        self.buf = torch.empty(nbytes + GUARD, dtype=torch.uint8, device=dev)
        self.buf[:nbytes].fill_(body)
        self.buf[nbytes:].fill_(CANARY)

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def bf16(self, shape):
        return self.buf[: self.nbytes].view(torch.bfloat16).view(*shape)

    def guard_ok(self) -> bool:
        return bool((self.buf[self.nbytes:] == CANARY).all())


def run_mlp(cfg, inp, w, X, dOut, body):
    dev = X.device
    N, d, f, r = cfg.N, cfg.d, cfg.d_ff, cfg.r
    shape = w.shape(N)
    fws, bws, svs = _lib.sizes(shape)
    out = Carved(N * d * 2, body, dev)
    g = Carved(N * f * 2, body, dev)
    u = Carved(N * f * 2, body, dev)
    saved = Carved(svs, body, dev)
    wsf = Carved(fws, body, dev)
    dX = Carved(N * d * 2, body, dev)
    grads = {}
    for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"):
        grads["d" + k] = Carved(getattr(w, k).numel() * 2, body, dev)
    wsb = Carved(bws, body, dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    _lib.check(_lib.forward(shape, w.c_struct(), ctypes.c_void_p(X.data_ptr()), out.ptr(), g.ptr(), u.ptr(),
                            saved.ptr(), wsf.ptr(), fws, stream), "lora_mlp_forward")
    gs = _lib.Grads(*[grads[k].buf.data_ptr() for k in _lib.GRAD_FIELDS])
    _lib.check(_lib.backward(shape, w.c_struct(), ctypes.c_void_p(X.data_ptr()), g.ptr(), u.ptr(), saved.ptr(),
                             ctypes.c_void_p(dOut.data_ptr()), dX.ptr(), gs, wsb.ptr(), bws, stream),
               "lora_mlp_backward")
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
    res = {"out": out.bf16((N, d)), "g": g.bf16((N, f)), "u": u.bf16((N, f)), "dX": dX.bf16((N, d))}
    for k, c in grads.items():
        res[k] = c.bf16(tuple(getattr(w, k[1:]).shape))
    carved = {"out": out, "g": g, "u": u, "saved": saved, "dX": dX, "ws_fwd": wsf, "ws_bwd": wsb, **grads}
    return res, carved


CASES = [
    synth.custom(300, 192, 320, 24, 8.0, seed_index=41),      # ragged N, r = 24
    synth.custom(130, 136, 200, 16, 32.0, seed_index=42),     # K and d_ff off the 64 grid
    synth.custom(1, 64, 128, 8, 16.0, seed_index=43),         # one token
    synth.custom(1000, 512, 1408, 64, 128.0, seed_index=44),  # several tiles in every dimension
    synth.custom(200, 256, 704, 16, 16.0, int4=True, seed_index=45),  # int4 frozen weights
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"N{c.N}_d{c.d}_dff{c.d_ff}_r{c.r}{'_int4' if c.int4 else ''}")
def test_every_output_written_nothing_past_it_and_no_stale_reads(cfg):
    inp = synth.make_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    nan_run, carved = run_mlp(cfg, inp, w, X, dOut, 0xFF)
    for k, t in nan_run.items():
        assert not torch.isnan(t).any(), f"{k}: elements left unwritten"
    for k, c in carved.items():
        assert c.guard_ok(), f"{k}: written past its end"
    zero_run, carved0 = run_mlp(cfg, inp, w, X, dOut, 0x00)
    for k in nan_run:
        assert torch.equal(nan_run[k].view(torch.int16), zero_run[k].view(torch.int16)), \
            f"{k}: depends on the buffers' initial contents"
    for k, c in carved0.items():
        assert c.guard_ok(), f"{k}: written past its end"


def test_lora_linear_writes_every_output_and_nothing_past_it():
    # ragged N, d_in and d_out off the 64 grid (d_out = 1.28 CTA-pair tiles)
    cfg = synth.LinearConfig("lin_guard", 300, 200, 328, 16, 32.0, index=46)
    inp = synth.make_linear_inputs(cfg)
    dev = torch.device("cuda:0")
    w = api.linear_weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dY = api.to_device_bf16(inp["dY"], dev)
    N = cfg.N
    shape = w.shape(N)
    runs = []
    for body in (0xFF, 0x00):
        fws, bws, svs = _lib.lin_sizes(shape)
        Y = Carved(N * cfg.d_out * 2, body, dev)
        saved = Carved(svs, body, dev)
        wsf = Carved(fws, body, dev)
        dX = Carved(N * cfg.d_in * 2, body, dev)
        dA = Carved(w.A.numel() * 2, body, dev)
        dB = Carved(w.B.numel() * 2, body, dev)
        wsb = Carved(bws, body, dev)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        _lib.check(_lib.lin_forward(shape, w.c_struct(), ctypes.c_void_p(X.data_ptr()), Y.ptr(), saved.ptr(),
                                    wsf.ptr(), fws, stream), "lora_linear_forward")
        _lib.check(_lib.lin_backward(shape, w.c_struct(), ctypes.c_void_p(X.data_ptr()), saved.ptr(),
                                     ctypes.c_void_p(dY.data_ptr()), dX.ptr(), dA.ptr(), dB.ptr(), wsb.ptr(), bws,
                                     stream), "lora_linear_backward")
        torch.cuda.synchronize()
        res = {"Y": Y.bf16((N, cfg.d_out)), "dX": dX.bf16((N, cfg.d_in)), "dA": dA.bf16(tuple(w.A.shape)),
               "dB": dB.bf16(tuple(w.B.shape))}
        for k, t in res.items():
            assert not torch.isnan(t).any(), f"{k}: elements left unwritten"
        for k, c in {"Y": Y, "saved": saved, "ws_fwd": wsf, "dX": dX, "dA": dA, "dB": dB, "ws_bwd": wsb}.items():
            assert c.guard_ok(), f"{k}: written past its end"
        runs.append(res)
    for k in runs[0]:
        assert torch.equal(runs[0][k].view(torch.int16), runs[1][k].view(torch.int16)), k


@pytest.mark.parametrize("name,ld_pad", [("ce_tiny", 5), ("ce_tiny_softcap", 0)])
def test_cross_entropy_writes_every_output_and_nothing_past_it(name, ld_pad):
    """loss and lse for every row, dlogits for every valid column (the padding
    columns of a row are not the kernel's), nothing past any buffer, and the
    same bits from poisoned and zeroed buffers."""
    import numpy as np

    cfg = synth.CE_BY_NAME[name]
    inp = synth.make_ce_inputs(cfg)
    N, V = inp["logits"].shape
    ld = (V + 7) // 8 * 8 + 8 * ld_pad
    dev = torch.device("cuda:0")
    z = torch.zeros((N, ld), dtype=torch.int16)
    z[:, :V] = torch.from_numpy(inp["logits"].view(np.int16))
    z = z.view(torch.bfloat16).to(dev)
    lab = torch.from_numpy(np.asarray(inp["labels"], dtype=np.int64)).to(dev)
    dl = torch.from_numpy(np.asarray(inp["dloss"], dtype=np.float32)).to(dev)
    shape = _lib.make_ce_shape(N, V, ld, cfg.logit_scale, cfg.softcap, synth.CE_IGNORE_INDEX)
    wsb = _lib.ce_sizes(shape)
    runs = []
    for body in (0xFF, 0x00):
        loss = Carved(N * 4, body, dev)
        lse = Carved(N * 4, body, dev)
        ws = Carved(wsb, body, dev)
        dz = Carved(N * ld * 2, body, dev)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        _lib.check(_lib.ce_forward(shape, ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(lab.data_ptr()),
                                   loss.ptr(), lse.ptr(), ws.ptr(), wsb, stream), "lora_ce_forward")
        _lib.check(_lib.ce_backward(shape, ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(lab.data_ptr()),
                                    lse.ptr(), ctypes.c_void_p(dl.data_ptr()), dz.ptr(), stream), "lora_ce_backward")
        torch.cuda.synchronize()
        res = {"loss": loss.buf[: N * 4].view(torch.float32), "dlogits": dz.bf16((N, ld))[:, :V]}
        valid = lab != synth.CE_IGNORE_INDEX
        res["lse"] = lse.buf[: N * 4].view(torch.float32)[valid]
        for k, t in res.items():
            assert not torch.isnan(t).any(), f"{k}: elements left unwritten"
        for k, c in {"loss": loss, "lse": lse, "workspace": ws, "dlogits": dz}.items():
            assert c.guard_ok(), f"{k}: written past its end"
        runs.append({k: v.clone() for k, v in res.items()})
    for k in runs[0]:
        assert torch.equal(runs[0][k].view(torch.int16) if runs[0][k].dtype == torch.bfloat16 else runs[0][k],
                           runs[1][k].view(torch.int16) if runs[1][k].dtype == torch.bfloat16 else runs[1][k]), k


def test_rmsnorm_writes_every_output_and_nothing_past_it():
    import numpy as np

    dev = torch.device("cuda:0")
    rng = np.random.default_rng(47)
    for N, d in ((3, 136), (257, 4096), (5, 20480)):   # one-row-per-CTA and wide-row kernels
        x = torch.from_numpy(rng.standard_normal((N, d)).astype(np.float32)).to(torch.bfloat16).to(dev)
        gamma = torch.from_numpy(rng.uniform(0.5, 1.5, d).astype(np.float32)).to(torch.bfloat16).to(dev)
        dy = torch.from_numpy(rng.standard_normal((N, d)).astype(np.float32)).to(torch.bfloat16).to(dev)
        runs = []
        for body in (0xFF, 0x00):
            y = Carved(N * d * 2, body, dev)
            rstd = Carved(N * 4, body, dev)
            dx = Carved(N * d * 2, body, dev)
            stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
            _lib.check(_lib.rmsnorm_forward(N, d, 1e-5, p(x), p(gamma), y.ptr(), rstd.ptr(), stream),
                       "lora_rmsnorm_forward")
            _lib.check(_lib.rmsnorm_backward(N, d, p(x), p(gamma), rstd.ptr(), p(dy), dx.ptr(), stream),
                       "lora_rmsnorm_backward")
            torch.cuda.synchronize()
            res = {"y": y.bf16((N, d)), "rstd": rstd.buf[: N * 4].view(torch.float32), "dx": dx.bf16((N, d))}
            for k, t in res.items():
                assert not torch.isnan(t).any(), f"{k} (N={N}, d={d}): elements left unwritten"
            for k, c in {"y": y, "rstd": rstd, "dx": dx}.items():
                assert c.guard_ok(), f"{k} (N={N}, d={d}): written past its end"
            runs.append({k: v.clone().view(torch.int32 if v.dtype == torch.float32 else torch.int16)
                         for k, v in res.items()})
        for k in runs[0]:
            assert torch.equal(runs[0][k], runs[1][k]), (k, N, d)


def test_host_memory_is_refused_before_any_launch():
    """The pointer check accepts device memory only; an entry point handed a
    host pointer returns LORA_MLP_ERR_INVALID_ARG without enqueueing work."""
    dev = torch.device("cuda:0")
    pageable = torch.zeros(4096, dtype=torch.uint8)
    pinned = torch.zeros(4096, dtype=torch.uint8).pin_memory()
    device = torch.zeros(4096, dtype=torch.uint8, device=dev)
    assert _lib.check_pointer(pageable.data_ptr(), 16) == _lib.ERR_INVALID_ARG
    assert _lib.check_pointer(pinned.data_ptr(), 16) == _lib.ERR_INVALID_ARG
    assert _lib.check_pointer(device.data_ptr(), 16) == _lib.OK
    assert _lib.check_pointer(device.data_ptr() + 8, 16) == _lib.ERR_MISALIGNED
    # an entry point given a host X (everything else on the device)
    cfg = synth.custom(64, 64, 128, 8, 16.0, seed_index=48)
    inp = synth.make_inputs(cfg)
    w = api.weights_from_host(inp, cfg.alpha, dev)
    shape = w.shape(cfg.N)
    fws, _, svs = _lib.sizes(shape)
    X_host = torch.zeros((cfg.N, cfg.d), dtype=torch.bfloat16).pin_memory()
    out = torch.empty((cfg.N, cfg.d), dtype=torch.bfloat16, device=dev)
    g = torch.empty((cfg.N, cfg.d_ff), dtype=torch.bfloat16, device=dev)
    u = torch.empty_like(g)
    saved = torch.empty(max(svs, 256), dtype=torch.uint8, device=dev)
    ws = torch.empty(max(fws, 256), dtype=torch.uint8, device=dev)
    before = _lib.launch_count()
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = _lib.forward(shape, w.c_struct(), p(X_host), p(out), p(g), p(u), p(saved), p(ws), ws.numel(),
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.ERR_INVALID_ARG
    assert _lib.launch_count() == before
    torch.cuda.synchronize()
    assert _lib.device_status(None) == 0
