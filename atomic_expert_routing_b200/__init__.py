"""Routed atomic-expert branch of an OmniMoE layer on B200 (sm_100a).

Thin binding over the C ABI of ``libomnimoe.so`` (include/omnimoe.h).  Every
step of the layer runs in the library's CUDA kernels; this module only checks
each tensor's placement, dtype and element count against the dims, allocates
outputs and workspace with PyTorch, and passes raw pointers and the current
CUDA stream.  There is no CPU path: calls need a CUDA
device and the built library and raise otherwise.

Names follow the layer: ``route`` (Cartesian Product Router), ``schedule``
(Expert-Centric Scheduling), ``expert_forward`` (grouped execution),
``moe_forward`` (all three), ``token_centric_forward`` (the ablation).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (OMNI_BF16, OMNI_F32, OMNI_FLAG_DENSE_TENSOR_CORES, OMNI_FLAG_ROUTER_SIMT,
                   OMNI_FLAG_STAGED_SMALL,
                   OMNI_WS_BACKWARD, OMNI_WS_EXPERT, OMNI_WS_FUSED,
                   OMNI_WS_ROUTE, OMNI_WS_SCHEDULE, OmniError)

__all__ = ["LayerDims", "route", "router_logits", "route_select", "schedule", "expert_forward", "moe_forward",
           "token_centric_forward", "new_counts", "OmniError", "workspace_size", "wait_selftest",
           "shared_mlp", "moe_mlp_forward", "mlp_workspace_size", "expert_forward_noalloc",
           "moe_forward_shard", "moe_forward_shard_routed", "cast_output", "moe_backward"]


@dataclass(frozen=True)
class LayerDims:
    L: int
    d: int
    Nr: int
    Nc: int
    k: int
    K: int
    B: int
    dtype: int = OMNI_BF16
    flags: int = 0

    @property
    def N(self) -> int:
        return self.Nr * self.Nc

    @property
    def M(self) -> int:
        return self.L * self.K

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == OMNI_F32 else torch.bfloat16

    def c(self) -> _lib.Dims:
        return _lib.Dims(self.L, self.d, self.Nr, self.Nc, self.k, self.K, self.B, self.dtype,
                         self.flags)

    @classmethod
    def of(cls, cfg, L=None, flags: int = 0) -> "LayerDims":
        """From any object with L, d, Nr, Nc, k, K, B, dtype attributes."""
        return cls(cfg.L if L is None else L, cfg.d, cfg.Nr, cfg.Nc, cfg.k, cfg.K, cfg.B,
                   cfg.dtype, flags)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the CUDA library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the CUDA library must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _device(*ts):
    for t in ts:
        if t is not None:
            return t.device
    raise ValueError("no tensor given")


def _expect(name, t, n, dtype, *, optional=False):
    """Refuse a tensor whose dtype differs from the one the call reads, or
    that holds fewer than the n elements the call touches.  The C ABI sees
    only pointers, so this is the one place a too-small buffer becomes an
    error instead of an out-of-bounds device access."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, the call reads {dtype}")
    if t.numel() < n:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {n}")


def _expect_io(D, **ts):
    """Checks by argument name: storage-type tensors (x, W, U, V, Wr, Wc, y),
    fp32 biases and logits, int32 counts."""
    f32, i32 = torch.float32, torch.int32
    spec = {
        "x": (D.L * D.d, D.torch_dtype), "y": (D.L * D.d, D.torch_dtype),
        "Wr": (D.Nr * D.d, D.torch_dtype), "Wc": (D.Nc * D.d, D.torch_dtype),
        "W": (D.N * D.d, D.torch_dtype), "V": (D.N * D.d, D.torch_dtype),
        "U": (D.N * D.d, D.torch_dtype),
        "bias_r": (D.Nr, f32), "bias_c": (D.Nc, f32),
        "logits": (D.L * (D.Nr + D.Nc), f32), "counts": (4, i32),
        "idx": (D.M, i32), "gate": (D.M, f32),
    }
    optional = {"bias_r", "bias_c", "counts", "y", "idx", "gate", "U"}
    for name, t in ts.items():
        n, dt = spec[name]
        _expect(name, t, n, dt, optional=name in optional)


def _expect_sched(D, sched):
    """A schedule passed to the grouped execution.  The execution does not
    read uniq, and reads group_off only up to the group count held on the
    device (counts[1] + 1 entries), so an exactly sized schedule is valid and
    only the task arrays' lengths are known on the host."""
    i32 = torch.int32
    for name, n, dt in (("task_token", D.M, i32), ("task_expert", D.M, i32),
                        ("task_gate", D.M, torch.float32), ("uniq", 0, i32),
                        ("group_off", 1, i32), ("counts", 4, i32)):
        if name not in sched:
            raise ValueError(f"schedule entry {name} is missing")
        _expect(name, sched[name], n, dt)


def workspace_size(D: LayerDims, which: int) -> int:
    n = C.c_size_t(0)
    dd = D.c()
    _lib.check("omni_workspace_size", _lib.load().omni_workspace_size(C.byref(dd), which,
                                                                       C.byref(n)))
    return int(n.value)


class Workspace:
    """Reusable device workspace (grows on demand)."""

    def __init__(self):
        self.buf = None

    def get(self, nbytes: int, device) -> torch.Tensor | None:
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        return self.buf


def _ws(D, which, device, ws):
    n = workspace_size(D, which)
    if ws is None:
        ws = Workspace()
    buf = ws.get(n, device)
    return (_ptr(buf) if buf is not None else None), n


def new_counts(device) -> torch.Tensor:
    """Zeroed int32[4] device counters: n_active, n_groups, status bits, reserved."""
    return torch.zeros(4, dtype=torch.int32, device=device)


def route(D: LayerDims, x, Wr, Wc, bias_r=None, bias_c=None, *, counts=None, ws=None,
          stream=None, with_score=True, out=None):
    """Cartesian Product Router: (idx int32 [L,K], gate f32 [L,K], score f32 [L,K] or None).
    out (optional): (idx, gate) tensors to write."""
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, bias_r=bias_r, bias_c=bias_c, counts=counts)
    dev = _device(x)
    if out is not None:
        idx, gate = out
        _expect_io(D, idx=idx, gate=gate)
    else:
        idx = torch.empty((D.L, D.K), dtype=torch.int32, device=dev)
        gate = torch.empty((D.L, D.K), dtype=torch.float32, device=dev)
    score = torch.empty((D.L, D.K), dtype=torch.float32, device=dev) if with_score else None
    wsp, n = _ws(D, OMNI_WS_ROUTE, dev, ws)
    dd = D.c()
    _lib.check("omni_route", _lib.load().omni_route(
        C.byref(dd), _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(bias_r), _ptr(bias_c), _ptr(idx),
        _ptr(gate), _ptr(score), _ptr(counts), wsp, n, _stream(stream)))
    return idx, gate, score


def router_logits(D: LayerDims, x, Wr, Wc, *, counts=None, ws=None, stream=None):
    """Router projections: float32 [L, Nr + Nc] (row logits, then column logits)."""
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, counts=counts)
    dev = _device(x)
    z = torch.empty((D.L, D.Nr + D.Nc), dtype=torch.float32, device=dev)
    wsp, n = _ws(D, OMNI_WS_ROUTE, dev, ws)
    dd = D.c()
    _lib.check("omni_router_logits", _lib.load().omni_router_logits(
        C.byref(dd), _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(z), _ptr(counts), wsp, n,
        _stream(stream)))
    return z


def route_select(D: LayerDims, logits, bias_r=None, bias_c=None, *, counts=None, stream=None):
    """Selection from axis logits [L, Nr + Nc] (float32)."""
    _expect_io(D, logits=logits, bias_r=bias_r, bias_c=bias_c, counts=counts)
    dev = _device(logits)
    idx = torch.empty((D.L, D.K), dtype=torch.int32, device=dev)
    gate = torch.empty((D.L, D.K), dtype=torch.float32, device=dev)
    score = torch.empty((D.L, D.K), dtype=torch.float32, device=dev)
    dd = D.c()
    _lib.check("omni_route_select", _lib.load().omni_route_select(
        C.byref(dd), _ptr(logits), _ptr(bias_r), _ptr(bias_c), _ptr(idx), _ptr(gate),
        _ptr(score), _ptr(counts), None, 0, _stream(stream)))
    return idx, gate, score


def schedule(D: LayerDims, idx, gate, *, counts=None, ws=None, stream=None) -> dict:
    """Expert-Centric Scheduling of the L*K routing decisions (device tensors)."""
    _expect_io(D, idx=idx, gate=gate, counts=counts)
    _expect("idx", idx, D.M, torch.int32)
    _expect("gate", gate, D.M, torch.float32)
    dev = _device(idx)
    M = D.M
    ucap = max(1, min(D.N, M))
    gmax = (ucap + D.B - 1) // D.B
    out = {
        "task_token": torch.empty(M, dtype=torch.int32, device=dev),
        "task_expert": torch.empty(M, dtype=torch.int32, device=dev),
        "task_gate": torch.empty(M, dtype=torch.float32, device=dev),
        "uniq": torch.empty(ucap, dtype=torch.int32, device=dev),
        "group_off": torch.empty(gmax + 1, dtype=torch.int32, device=dev),
        "counts": new_counts(dev) if counts is None else counts,
    }
    wsp, n = _ws(D, OMNI_WS_SCHEDULE, dev, ws)
    dd = D.c()
    _lib.check("omni_schedule", _lib.load().omni_schedule(
        C.byref(dd), _ptr(idx), _ptr(gate), _ptr(out["task_token"]), _ptr(out["task_expert"]),
        _ptr(out["task_gate"]), _ptr(out["uniq"]), _ptr(out["group_off"]), _ptr(out["counts"]),
        wsp, n, _stream(stream)))
    return out


def _weights(fn, W, U, V):
    """The entry point and the expert-weight pointers: the plain expert
    (W, V), or with U the gated one, h = SiLU(x.W[e]) * (x.U[e])."""
    if U is None:
        return fn, (_ptr(W), _ptr(V))
    return fn + "_glu", (_ptr(W), _ptr(U), _ptr(V))


def expert_forward(D: LayerDims, x, W, V, sched: dict, *, U=None, y=None, ws=None,
                   stream=None):
    """Grouped (expert-centric) execution of a schedule; returns y [L, d].
    U [N, d] (optional): the gate matrix of gated (SwiGLU) experts."""
    _expect_io(D, x=x, W=W, U=U, V=V, y=y)
    _expect_sched(D, sched)
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    wsp, n = _ws(D, OMNI_WS_EXPERT, dev, ws)
    dd = D.c()
    fn, wts = _weights("omni_expert_forward", W, U, V)
    _lib.check(fn, getattr(_lib.load(), fn)(
        C.byref(dd), _ptr(x), *wts, _ptr(sched["task_token"]),
        _ptr(sched["task_expert"]), _ptr(sched["task_gate"]), _ptr(sched["uniq"]),
        _ptr(sched["group_off"]), _ptr(sched["counts"]), _ptr(y), wsp, n, _stream(stream)))
    return y


def expert_forward_noalloc(D: LayerDims, x, W, V, sched: dict, *, y=None, stream=None):
    """Grouped execution without a workspace, for callers that cannot allocate
    device memory when the layer runs (the accumulator is a fixed array inside
    the library; L*d <= 4194304; calls must not overlap on the GPU).  Pass y to
    keep the call itself free of allocations."""
    _expect_io(D, x=x, W=W, V=V, y=y)
    _expect_sched(D, sched)
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    dd = D.c()
    args = (_ptr(x), _ptr(W), _ptr(V), _ptr(sched["task_token"]), _ptr(sched["task_expert"]),
            _ptr(sched["task_gate"]), _ptr(sched["uniq"]), _ptr(sched["group_off"]),
            _ptr(sched["counts"]), _ptr(y))
    # the library uses the fixed array of the current device
    with torch.cuda.device(dev):
        _lib.check("omni_expert_forward_noalloc", _lib.load().omni_expert_forward_noalloc(
            C.byref(dd), *args, _stream(stream)))
    return y


def moe_forward(D: LayerDims, x, Wr, Wc, W, V, bias_r=None, bias_c=None, *, U=None, y=None,
                counts=None, idx=None, gate=None, ws=None, stream=None):
    """Route -> schedule -> grouped execution in one call; returns y [L, d].
    U [N, d] (optional): the gate matrix of gated (SwiGLU) experts."""
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, W=W, U=U, V=V, bias_r=bias_r, bias_c=bias_c, y=y,
               counts=counts, idx=idx, gate=gate)
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    if counts is None:
        counts = new_counts(dev)
    wsp, n = _ws(D, OMNI_WS_FUSED, dev, ws)
    dd = D.c()
    fn, wts = _weights("omni_moe_forward", W, U, V)
    _lib.check(fn, getattr(_lib.load(), fn)(
        C.byref(dd), _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(bias_r), _ptr(bias_c), *wts,
        _ptr(y), _ptr(idx), _ptr(gate), _ptr(counts), wsp, n, _stream(stream)))
    return y


def moe_forward_shard(D: LayerDims, x, Wr, Wc, W, V, e_lo: int, e_hi: int, bias_r=None,
                      bias_c=None, *, U=None, y_part=None, counts=None, idx=None, gate=None,
                      ws=None, stream=None):
    """This process' share of an expert-sharded forward: routing over all N
    ids, execution of the tasks whose expert lies in [e_lo, e_hi) only, with
    W, V (and U) the shard's rows [(e_hi - e_lo), d].  Returns y_part [L, d]
    fp32, the shard's partial sum (add the shards' partials, then
    cast_output)."""
    if not 0 <= e_lo < e_hi <= D.N:
        raise ValueError(f"shard ids [{e_lo}, {e_hi}) outside [0, {D.N})")
    rows = (e_hi - e_lo) * D.d
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, bias_r=bias_r, bias_c=bias_c, counts=counts, idx=idx,
               gate=gate)
    for name, t in (("W", W), ("V", V), ("U", U)):
        _expect(name, t, rows, D.torch_dtype, optional=name == "U")
    _expect("y_part", y_part, D.L * D.d, torch.float32, optional=True)
    dev = _device(x)
    if y_part is None:
        y_part = torch.empty((D.L, D.d), dtype=torch.float32, device=dev)
    if counts is None:
        counts = new_counts(dev)
    wsp, n = _ws(D, OMNI_WS_FUSED, dev, ws)
    dd = D.c()
    _lib.check("omni_moe_forward_shard", _lib.load().omni_moe_forward_shard(
        C.byref(dd), e_lo, e_hi, _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(bias_r), _ptr(bias_c),
        _ptr(W), _ptr(U), _ptr(V), _ptr(y_part), _ptr(idx), _ptr(gate), _ptr(counts), wsp, n,
        _stream(stream)))
    return y_part


def moe_forward_shard_routed(D: LayerDims, x, W, V, e_lo: int, e_hi: int, idx, gate, *,
                             U=None, y_part=None, counts=None, ws=None, stream=None):
    """moe_forward_shard from a given routing (idx, gate [L, K] of all L
    tokens), which is read and not computed.  Returns y_part [L, d] fp32."""
    if not 0 <= e_lo < e_hi <= D.N:
        raise ValueError(f"shard ids [{e_lo}, {e_hi}) outside [0, {D.N})")
    rows = (e_hi - e_lo) * D.d
    _expect_io(D, x=x, counts=counts)
    _expect("idx", idx, D.M, torch.int32)
    _expect("gate", gate, D.M, torch.float32)
    for name, t in (("W", W), ("V", V), ("U", U)):
        _expect(name, t, rows, D.torch_dtype, optional=name == "U")
    _expect("y_part", y_part, D.L * D.d, torch.float32, optional=True)
    dev = _device(x)
    if y_part is None:
        y_part = torch.empty((D.L, D.d), dtype=torch.float32, device=dev)
    if counts is None:
        counts = new_counts(dev)
    wsp, n = _ws(D, OMNI_WS_FUSED, dev, ws)
    dd = D.c()
    _lib.check("omni_moe_forward_shard_routed", _lib.load().omni_moe_forward_shard_routed(
        C.byref(dd), e_lo, e_hi, _ptr(x), _ptr(W), _ptr(U), _ptr(V), _ptr(idx), _ptr(gate),
        _ptr(y_part), _ptr(counts), wsp, n, _stream(stream)))
    return y_part


def cast_output(D: LayerDims, src, *, y=None, stream=None):
    """y [L, d] in the storage type from an fp32 [L, d] sum (bf16: nearest even)."""
    _expect("src", src, D.L * D.d, torch.float32)
    _expect_io(D, y=y)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=_device(src))
    dd = D.c()
    _lib.check("omni_cast_output", _lib.load().omni_cast_output(
        C.byref(dd), _ptr(src), _ptr(y), _stream(stream)))
    return y


def moe_backward(D: LayerDims, x, Wr, Wc, W, V, idx, gate, dy, *, grads=None, bias=True,
                 accumulate=True, counts=None, ws=None, stream=None):
    """Gradients of the loss sum(dy * y) with the forward's routing (idx,
    gate) fixed.  grads (optional): a dict of fp32 tensors for the parameter
    gradients -- dW, dV [N, d], dWr [Nr, d], dWc [Nc, d], dbias_r [Nr],
    dbias_c [Nc] (missing ones are created as zeros; with bias=False the bias
    gradients are skipped), added to (accumulate) or overwritten (rows of
    dW, dV of experts no token chose untouched either way) -- and dx [L, d]
    (fp32, overwritten).  Returns the dict."""
    f32 = torch.float32
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, W=W, V=V, idx=idx, gate=gate, counts=counts)
    _expect("dy", dy, D.L * D.d, D.torch_dtype)
    dev = _device(x)
    shapes = {"dx": (D.L, D.d), "dW": (D.N, D.d), "dV": (D.N, D.d), "dWr": (D.Nr, D.d),
              "dWc": (D.Nc, D.d), "dbias_r": (D.Nr,), "dbias_c": (D.Nc,)}
    g = dict(grads or {})
    for name, shape in shapes.items():
        if name.startswith("dbias") and not bias:
            g.pop(name, None)
            continue
        if name not in g:
            g[name] = (torch.empty if name == "dx" else torch.zeros)(shape, dtype=f32, device=dev)
        n = 1
        for v in shape:
            n *= v
        _expect(name, g[name], n, f32)
    if counts is None:
        counts = new_counts(dev)
    wsp, n = _ws(D, OMNI_WS_BACKWARD, dev, ws)
    dd = D.c()
    _lib.check("omni_moe_backward", _lib.load().omni_moe_backward(
        C.byref(dd), _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(W), _ptr(V), _ptr(idx), _ptr(gate),
        _ptr(dy), _ptr(g["dx"]), _ptr(g["dW"]), _ptr(g["dV"]), _ptr(g["dWr"]), _ptr(g["dWc"]),
        _ptr(g.get("dbias_r")), _ptr(g.get("dbias_c")), 1 if accumulate else 0, _ptr(counts),
        wsp, n, _stream(stream)))
    return g


def mlp_workspace_size(D: LayerDims, F: int, with_routed: bool) -> int:
    n = C.c_size_t(0)
    dd = D.c()
    _lib.check("omni_mlp_workspace_size", _lib.load().omni_mlp_workspace_size(
        C.byref(dd), C.c_int64(F), 1 if with_routed else 0, C.byref(n)))
    return int(n.value)


def _expect_mlp(D, F, W1, W2):
    _expect("W1", W1, F * D.d, D.torch_dtype)
    _expect("W2", W2, D.d * F, D.torch_dtype)


def shared_mlp(D: LayerDims, x, W1, W2, *, y=None, accumulate=False, counts=None, ws=None,
               stream=None):
    """Shared dense MLP branch: y (+)= SiLU(x W1^T) W2^T (W1 [F, d], W2 [d, F], bf16)."""
    F = int(W1.shape[0])
    _expect_io(D, x=x, y=y, counts=counts)
    _expect_mlp(D, F, W1, W2)
    if accumulate and y is None:
        raise ValueError("y is required to accumulate into")
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    n = mlp_workspace_size(D, F, False)
    buf = (Workspace() if ws is None else ws).get(n, dev)
    dd = D.c()
    _lib.check("omni_shared_mlp", _lib.load().omni_shared_mlp(
        C.byref(dd), C.c_int64(F), _ptr(x), _ptr(W1), _ptr(W2), _ptr(y), 1 if accumulate else 0,
        _ptr(counts), _ptr(buf) if buf is not None else None, n, _stream(stream)))
    return y


def moe_mlp_forward(D: LayerDims, x, Wr, Wc, W, V, W1, W2, bias_r=None, bias_c=None, *, y=None,
                    counts=None, idx=None, gate=None, ws=None, stream=None):
    """The layer output routed(x) + MLP(x) in one call; returns y [L, d]."""
    F = int(W1.shape[0])
    _expect_io(D, x=x, Wr=Wr, Wc=Wc, W=W, V=V, bias_r=bias_r, bias_c=bias_c, y=y,
               counts=counts, idx=idx, gate=gate)
    _expect_mlp(D, F, W1, W2)
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    if counts is None:
        counts = new_counts(dev)
    n = mlp_workspace_size(D, F, True)
    buf = (Workspace() if ws is None else ws).get(n, dev)
    dd = D.c()
    _lib.check("omni_moe_mlp_forward", _lib.load().omni_moe_mlp_forward(
        C.byref(dd), C.c_int64(F), _ptr(x), _ptr(Wr), _ptr(Wc), _ptr(bias_r), _ptr(bias_c),
        _ptr(W), _ptr(V), _ptr(W1), _ptr(W2), _ptr(y), _ptr(idx), _ptr(gate), _ptr(counts),
        _ptr(buf) if buf is not None else None, n, _stream(stream)))
    return y


def token_centric_forward(D: LayerDims, x, W, V, idx, gate, *, U=None, y=None, counts=None,
                          stream=None):
    """Token-centric execution (ablation): every token gathers its own experts.
    U [N, d] (optional): the gate matrix of gated (SwiGLU) experts."""
    _expect_io(D, x=x, W=W, U=U, V=V, y=y, counts=counts)
    _expect("idx", idx, D.M, torch.int32)
    _expect("gate", gate, D.M, torch.float32)
    dev = _device(x)
    if y is None:
        y = torch.empty((D.L, D.d), dtype=D.torch_dtype, device=dev)
    dd = D.c()
    fn, wts = _weights("omni_token_centric_forward", W, U, V)
    _lib.check(fn, getattr(_lib.load(), fn)(
        C.byref(dd), _ptr(x), *wts, _ptr(idx), _ptr(gate), _ptr(y), _ptr(counts),
        None, 0, _stream(stream)))
    return y


def wait_selftest(counts, *, stream=None):
    """Makes one bounded device wait run out (about 1 s): afterwards counts[2]
    holds OMNI_DEV_TIMEOUT.  A check of the failure reporting, not a layer op."""
    _expect("counts", counts, 4, torch.int32)
    _device(counts)
    _lib.check("omni_wait_selftest", _lib.load().omni_wait_selftest(_ptr(counts),
                                                                    _stream(stream)))
