"""Python access to the fp64 CPU oracle (``oracle.c``) of the routed atomic-expert layer.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package and this package never imports the product library.

Arguments are numpy arrays laid out as in ``workloads`` (bf16 stored as uint16
bits).  A token subset ``tokens`` (sorted int64 ids) restricts routing and
execution to those tokens; outputs then have one row per listed token.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class _Dims(C.Structure):
    _fields_ = [("L", C.c_int64), ("d", C.c_int64), ("Nr", C.c_int64), ("Nc", C.c_int64),
                ("k", C.c_int64), ("K", C.c_int64), ("B", C.c_int64), ("dtype", C.c_int32),
                ("pad", C.c_int32)]


def lib():
    """The oracle's shared library.  ``OMNI_ORACLE_LIB`` names another build of
    ``oracle.c`` instead: the mutation tests run the pins against copies with
    one planted mistake each, loaded this way in a child process."""
    global _lib
    if _lib is None:
        _lib = C.CDLL(os.environ.get("OMNI_ORACLE_LIB") or _build.build())
        _lib.oracle_num_threads.restype = C.c_int
    return _lib


def dims(cfg) -> _Dims:
    return _Dims(cfg.L, cfg.d, cfg.Nr, cfg.Nc, cfg.k, cfg.K, cfg.B, cfg.dtype, 0)


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's later OpenMP regions (timing only)."""
    lib().oracle_set_num_threads(C.c_int(int(n)))


def _tokens(cfg, tokens):
    if tokens is None:
        return np.arange(cfg.L, dtype=np.int64)
    return np.ascontiguousarray(tokens, dtype=np.int64)


def axis_logits(cfg, inp, tokens=None):
    """Raw router logits (zr [nt, Nr], zc [nt, Nc]) including the optional biases."""
    tok = _tokens(cfg, tokens)
    zr = np.empty((len(tok), cfg.Nr), np.float64)
    zc = np.empty((len(tok), cfg.Nc), np.float64)
    br = None if inp.get("bias_r") is None else np.ascontiguousarray(inp["bias_r"], np.float32)
    bc = None if inp.get("bias_c") is None else np.ascontiguousarray(inp["bias_c"], np.float32)
    D = dims(cfg)
    _check(lib().oracle_axis_logits(C.byref(D), _p(inp["x"]), _p(inp["Wr"]), _p(inp["Wc"]),
                                    _p(br), _p(bc), _p(tok), C.c_int64(len(tok)), _p(zr),
                                    _p(zc)), "axis_logits")
    return zr, zc


def axis_logprobs(cfg, inp, tokens=None):
    """Per-axis log-softmax of the router logits: (lr [nt, Nr], lc [nt, Nc])."""
    tok = _tokens(cfg, tokens)
    lr = np.empty((len(tok), cfg.Nr), np.float64)
    lc = np.empty((len(tok), cfg.Nc), np.float64)
    br = None if inp.get("bias_r") is None else np.ascontiguousarray(inp["bias_r"], np.float32)
    bc = None if inp.get("bias_c") is None else np.ascontiguousarray(inp["bias_c"], np.float32)
    D = dims(cfg)
    _check(lib().oracle_axis_logprobs(C.byref(D), _p(inp["x"]), _p(inp["Wr"]), _p(inp["Wc"]),
                                      _p(br), _p(bc), _p(tok), C.c_int64(len(tok)), _p(lr),
                                      _p(lc)), "axis_logprobs")
    return lr, lc


def log_softmax(z):
    """Row-wise log-softmax of float64 logits (returns a new array)."""
    z = np.array(z, dtype=np.float64, order="C", copy=True)
    lib().oracle_log_softmax(_p(z), C.c_int64(z.shape[0]), C.c_int64(z.shape[1]))
    return z


def select(cfg, lr, lc):
    """k x k-candidate selection: idx [nt, K] int32, gate, score [nt, K] float64."""
    lr = np.ascontiguousarray(lr, np.float64)
    lc = np.ascontiguousarray(lc, np.float64)
    nt = lr.shape[0]
    idx = np.empty((nt, cfg.K), np.int32)
    gate = np.empty((nt, cfg.K), np.float64)
    score = np.empty((nt, cfg.K), np.float64)
    D = dims(cfg)
    _check(lib().oracle_select(C.byref(D), _p(lr), _p(lc), C.c_int64(nt), _p(idx), _p(gate),
                               _p(score)), "select")
    return idx, gate, score


def select_bruteforce(cfg, lr, lc):
    """Selection over all N joint scores: idx, gate, score and the (K+1)-th score."""
    lr = np.ascontiguousarray(lr, np.float64)
    lc = np.ascontiguousarray(lc, np.float64)
    nt = lr.shape[0]
    idx = np.empty((nt, cfg.K), np.int32)
    gate = np.empty((nt, cfg.K), np.float64)
    score = np.empty((nt, cfg.K), np.float64)
    nxt = np.empty(nt, np.float64)
    D = dims(cfg)
    _check(lib().oracle_select_bruteforce(C.byref(D), _p(lr), _p(lc), C.c_int64(nt), _p(idx),
                                          _p(gate), _p(score), _p(nxt)), "select_bruteforce")
    return idx, gate, score, nxt


def route(cfg, inp, tokens=None):
    lr, lc = axis_logprobs(cfg, inp, tokens)
    return select(cfg, lr, lc)


def schedule(cfg, idx, gate, tokens=None):
    """Expert-centric schedule of the tasks of the listed tokens (dict of arrays)."""
    tok = _tokens(cfg, tokens)
    idx = np.ascontiguousarray(idx, np.int32)
    gate = np.ascontiguousarray(gate, np.float64)
    M = len(tok) * cfg.K
    ucap = max(1, min(cfg.N, M))
    out = {
        "task_token": np.empty(M, np.int32),
        "task_expert": np.empty(M, np.int32),
        "task_gate": np.empty(M, np.float64),
        "uniq": np.empty(ucap, np.int32),
        "group_off": np.empty((ucap + cfg.B - 1) // cfg.B + 1, np.int32),
    }
    na = C.c_int64(0)
    ng = C.c_int64(0)
    D = dims(cfg)
    _check(lib().oracle_schedule(C.byref(D), _p(tok), C.c_int64(len(tok)), _p(idx), _p(gate),
                                 _p(out["task_token"]), _p(out["task_expert"]),
                                 _p(out["task_gate"]), _p(out["uniq"]), _p(out["group_off"]),
                                 C.byref(na), C.byref(ng)), "schedule")
    out["n_active"] = int(na.value)
    out["n_groups"] = int(ng.value)
    out["uniq"] = out["uniq"][: out["n_active"]]
    out["group_off"] = out["group_off"][: out["n_groups"] + 1]
    return out


def forward_expert(cfg, inp, sched, tokens=None):
    """Expert-centric execution; returns (y [nt, d] float64, rows_loaded (W, V)).
    With inp["U"] the experts are gated: h = SiLU(x.W[e]) * (x.U[e])."""
    tok = _tokens(cfg, tokens)
    out_row = np.full(cfg.L, -1, np.int64)
    out_row[tok] = np.arange(len(tok))
    y = np.empty((len(tok), cfg.d), np.float64)
    rows = np.zeros(2, np.int64)
    D = dims(cfg)
    go = np.ascontiguousarray(sched["group_off"], np.int32)
    _check(lib().oracle_forward_expert(
        C.byref(D), _p(inp["x"]), _p(inp["W"]), _p(inp.get("U")), _p(inp["V"]),
        _p(np.ascontiguousarray(sched["task_token"], np.int32)),
        _p(np.ascontiguousarray(sched["task_expert"], np.int32)),
        _p(np.ascontiguousarray(sched["task_gate"], np.float64)),
        _p(np.ascontiguousarray(sched["uniq"], np.int32)), _p(go),
        C.c_int64(sched["n_active"]), C.c_int64(sched["n_groups"]), _p(out_row), _p(y),
        C.c_int64(len(tok)), _p(rows)), "forward_expert")
    return y, (int(rows[0]), int(rows[1]))


def forward_token(cfg, inp, idx, gate, tokens=None):
    """Token-centric execution; returns (y [nt, d] float64, rows_loaded (W, V)).
    With inp["U"] the experts are gated, as in forward_expert."""
    tok = _tokens(cfg, tokens)
    y = np.empty((len(tok), cfg.d), np.float64)
    rows = np.zeros(2, np.int64)
    D = dims(cfg)
    _check(lib().oracle_forward_token(
        C.byref(D), _p(inp["x"]), _p(inp["W"]), _p(inp.get("U")), _p(inp["V"]), _p(tok),
        C.c_int64(len(tok)),
        _p(np.ascontiguousarray(idx, np.int32)), _p(np.ascontiguousarray(gate, np.float64)),
        _p(y), _p(rows)), "forward_token")
    return y, (int(rows[0]), int(rows[1]))


def moe_forward(cfg, inp, tokens=None):
    """Route -> schedule -> expert-centric execution for the listed tokens."""
    idx, gate, score = route(cfg, inp, tokens)
    sched = schedule(cfg, idx, gate, tokens)
    y, rows = forward_expert(cfg, inp, sched, tokens)
    return {"idx": idx, "gate": gate, "score": score, "sched": sched, "y": y, "rows": rows}


def backward(cfg, inp, idx, gate, dy, tokens=None):
    """Gradients of the routed branch for the loss sum(dy * y), with the
    forward's routing (idx, gate) fixed; dy [nt, d] float64.  Returns a dict
    of float64 arrays: dx [nt, d], dW, dV [N, d], dWr [Nr, d], dWc [Nc, d],
    dbias_r [Nr], dbias_c [Nc] (the parameter gradients of these tokens
    alone)."""
    tok = _tokens(cfg, tokens)
    nt = len(tok)
    out = {"dx": np.empty((nt, cfg.d), np.float64),
           "dW": np.zeros((cfg.N, cfg.d), np.float64), "dV": np.zeros((cfg.N, cfg.d), np.float64),
           "dWr": np.zeros((cfg.Nr, cfg.d), np.float64),
           "dWc": np.zeros((cfg.Nc, cfg.d), np.float64),
           "dbias_r": np.zeros(cfg.Nr, np.float64), "dbias_c": np.zeros(cfg.Nc, np.float64)}
    D = dims(cfg)
    br = None if inp.get("bias_r") is None else np.ascontiguousarray(inp["bias_r"], np.float32)
    bc = None if inp.get("bias_c") is None else np.ascontiguousarray(inp["bias_c"], np.float32)
    _check(lib().oracle_backward(
        C.byref(D), _p(inp["x"]), _p(inp["Wr"]), _p(inp["Wc"]), _p(br), _p(bc), _p(inp["W"]),
        _p(inp["V"]), _p(tok), C.c_int64(nt),
        _p(np.ascontiguousarray(idx, np.int32)), _p(np.ascontiguousarray(gate, np.float64)),
        _p(np.ascontiguousarray(dy, np.float64)), _p(out["dx"]), _p(out["dW"]), _p(out["dV"]),
        _p(out["dWr"]), _p(out["dWc"]), _p(out["dbias_r"]), _p(out["dbias_c"])), "backward")
    return out


def shared_mlp(cfg, inp, W1, W2, tokens=None):
    """The shared dense MLP branch: SiLU(x W1^T) W2^T, fp64 [nt, d].  W1 [F, d]
    and W2 [d, F] in the storage layout of ``workloads`` (bf16 as uint16)."""
    tok = _tokens(cfg, tokens)
    W1 = np.ascontiguousarray(W1)
    W2 = np.ascontiguousarray(W2)
    F = W1.shape[0]
    assert W1.shape == (F, cfg.d) and W2.shape == (cfg.d, F)
    y = np.empty((len(tok), cfg.d), np.float64)
    D = dims(cfg)
    _check(lib().oracle_shared_mlp(C.byref(D), C.c_int64(F), _p(inp["x"]), _p(W1), _p(W2),
                                   _p(tok), C.c_int64(len(tok)), _p(y)), "shared_mlp")
    return y
