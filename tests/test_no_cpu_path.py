"""The product has no CPU path: every compute entry of the binding refuses
host tensors before the library is asked to run anything, a missing library
is an error, and the product package never imports the oracle."""
import ast
import glob
import os
import subprocess
import sys

import pytest
import torch

import atomic_expert_routing_b200 as omni
import workloads as WL
from atomic_expert_routing_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = WL.Config("host", L=8, d=64, Nr=8, Nc=8, k=2, K=2, B=2, dtype=WL.F32)


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


def _calls():
    c = CFG
    D = omni.LayerDims.of(c)
    x, Wr, Wc = _t(c.L, c.d), _t(c.Nr, c.d), _t(c.Nc, c.d)
    W, V = _t(c.N, c.d), _t(c.N, c.d)
    idx = torch.zeros((c.L, c.K), dtype=torch.int32)
    gate = _t(c.L, c.K)
    M = c.L * c.K
    sched = {"task_token": torch.zeros(M, dtype=torch.int32),
             "task_expert": torch.zeros(M, dtype=torch.int32), "task_gate": _t(M),
             "uniq": torch.zeros(M, dtype=torch.int32),
             "group_off": torch.zeros(M + 1, dtype=torch.int32),
             "counts": torch.zeros(4, dtype=torch.int32)}
    return {
        "route": lambda: omni.route(D, x, Wr, Wc),
        "router_logits": lambda: omni.router_logits(D, x, Wr, Wc),
        "route_select": lambda: omni.route_select(D, _t(c.L, c.Nr + c.Nc)),
        "schedule": lambda: omni.schedule(D, idx, gate),
        "expert_forward": lambda: omni.expert_forward(D, x, W, V, sched),
        "expert_forward_noalloc": lambda: omni.expert_forward_noalloc(D, x, W, V, sched),
        "moe_forward": lambda: omni.moe_forward(D, x, Wr, Wc, W, V),
        "token_centric_forward": lambda: omni.token_centric_forward(D, x, W, V, idx, gate),
        "moe_forward-glu": lambda: omni.moe_forward(D, x, Wr, Wc, W, V, U=W),
        "expert_forward-glu": lambda: omni.expert_forward(D, x, W, V, sched, U=W),
        "token_centric_forward-glu":
            lambda: omni.token_centric_forward(D, x, W, V, idx, gate, U=W),
        "moe_forward_shard": lambda: omni.moe_forward_shard(D, x, Wr, Wc, W[:2], V[:2], 0, 2),
        "cast_output": lambda: omni.cast_output(D, _t(c.L, c.d)),
        "wait_selftest": lambda: omni.wait_selftest(torch.zeros(4, dtype=torch.int32)),
    }


def _mlp_calls():
    c = CFG.with_(dtype=WL.BF16)
    D = omni.LayerDims.of(c)
    b = torch.bfloat16
    x, Wr, Wc = _t(c.L, c.d, dtype=b), _t(c.Nr, c.d, dtype=b), _t(c.Nc, c.d, dtype=b)
    W, V = _t(c.N, c.d, dtype=b), _t(c.N, c.d, dtype=b)
    W1, W2 = _t(16, c.d, dtype=b), _t(c.d, 16, dtype=b)
    return {
        "shared_mlp": lambda: omni.shared_mlp(D, x, W1, W2),
        "moe_mlp_forward": lambda: omni.moe_mlp_forward(D, x, Wr, Wc, W, V, W1, W2),
    }


@pytest.mark.parametrize("name", list(_calls()) + list(_mlp_calls()))
def test_host_tensors_are_refused(name):
    calls = dict(_calls(), **_mlp_calls())
    with pytest.raises(ValueError, match="CUDA device"):
        calls[name]()


def test_a_missing_library_is_an_error(tmp_path):
    """In a fresh process (the loaded library is cached per process)."""
    missing = str(tmp_path / "libomnimoe.so")
    r = subprocess.run([sys.executable, "-c",
                        "from atomic_expert_routing_b200 import _lib; _lib.load(%r)" % missing],
                       cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0
    assert "RuntimeError" in r.stderr and "is missing" in r.stderr


def test_the_product_never_imports_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "atomic_expert_routing_b200", "*.py")):
        tree = ast.parse(open(path).read())
        for node in ast.walk(tree):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), path


def _shrunk_calls():
    """Each compute entry with one argument a row too short or of the wrong
    dtype: (call name, argument name, call)."""
    c = CFG
    D = omni.LayerDims.of(c)
    M = c.L * c.K
    x, Wr, Wc = _t(c.L, c.d), _t(c.Nr, c.d), _t(c.Nc, c.d)
    W, V = _t(c.N, c.d), _t(c.N, c.d)
    idx = torch.zeros((c.L, c.K), dtype=torch.int32)
    gate = _t(c.L, c.K)
    sched = {"task_token": torch.zeros(M, dtype=torch.int32),
             "task_expert": torch.zeros(M, dtype=torch.int32), "task_gate": _t(M),
             "uniq": torch.zeros(M, dtype=torch.int32),
             "group_off": torch.zeros(M + 1, dtype=torch.int32),
             "counts": torch.zeros(4, dtype=torch.int32)}
    short = dict(sched, task_expert=torch.zeros(M - 1, dtype=torch.int32))
    return [
        ("route", "x", lambda: omni.route(D, x[:-1], Wr, Wc)),
        ("route", "Wc", lambda: omni.route(D, x, Wr, Wc.to(torch.float64))),
        ("route", "bias_r", lambda: omni.route(D, x, Wr, Wc, bias_r=_t(c.Nr - 1))),
        ("router_logits", "Wr", lambda: omni.router_logits(D, x, Wr[:-1], Wc)),
        ("route_select", "logits", lambda: omni.route_select(D, _t(c.L - 1, c.Nr + c.Nc))),
        ("schedule", "idx", lambda: omni.schedule(D, idx.long(), gate)),
        ("schedule", "gate", lambda: omni.schedule(D, idx, gate[:-1])),
        ("expert_forward", "W", lambda: omni.expert_forward(D, x, W[:-1], V, sched)),
        ("expert_forward", "task_expert", lambda: omni.expert_forward(D, x, W, V, short)),
        ("expert_forward", "y", lambda: omni.expert_forward(D, x, W, V, sched, y=_t(1))),
        ("expert_forward_noalloc", "V",
         lambda: omni.expert_forward_noalloc(D, x, W, V.half(), sched)),
        ("moe_forward", "V", lambda: omni.moe_forward(D, x, Wr, Wc, W, V[:-1])),
        ("moe_forward", "counts",
         lambda: omni.moe_forward(D, x, Wr, Wc, W, V, counts=torch.zeros(3, dtype=torch.int32))),
        ("token_centric_forward", "gate",
         lambda: omni.token_centric_forward(D, x, W, V, idx, gate.double())),
        ("moe_forward", "U", lambda: omni.moe_forward(D, x, Wr, Wc, W, V, U=W[:-1])),
        ("expert_forward", "U", lambda: omni.expert_forward(D, x, W, V, sched, U=W.half())),
        ("token_centric_forward", "U",
         lambda: omni.token_centric_forward(D, x, W, V, idx, gate, U=W[:-1])),
        ("moe_forward_shard", "W",
         lambda: omni.moe_forward_shard(D, x, Wr, Wc, W[:1], V[:2], 0, 2)),
        ("moe_forward_shard", "y_part",
         lambda: omni.moe_forward_shard(D, x, Wr, Wc, W[:2], V[:2], 0, 2, y_part=x.half())),
        ("cast_output", "src", lambda: omni.cast_output(D, x.double())),
        ("cast_output", "y", lambda: omni.cast_output(D, x, y=x[:-1])),
        ("wait_selftest", "counts", lambda: omni.wait_selftest(torch.zeros(4))),
    ]


@pytest.mark.parametrize("case", _shrunk_calls(), ids=lambda c: f"{c[0]}-{c[1]}")
def test_sizes_and_dtypes_are_checked_before_the_library(case, monkeypatch):
    """A tensor too small for the dims, or of another dtype, raises in the
    binding; the library is never loaded or called."""
    def no_library(*a, **k):
        raise AssertionError("the library was reached")

    monkeypatch.setattr(_lib, "load", no_library)
    _, arg, call = case
    with pytest.raises(ValueError, match=rf"^{arg}\b"):
        call()
