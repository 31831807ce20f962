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
        "wait_selftest": lambda: omni.wait_selftest(torch.zeros(4, dtype=torch.int32)),
    }


@pytest.mark.parametrize("name", list(_calls()))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="CUDA device"):
        _calls()[name]()


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
