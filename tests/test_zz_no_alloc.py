"""omni_expert_forward_noalloc: the grouped execution for callers that cannot
allocate device memory while the layer runs (graph capture, ahead-of-time
memory plans, plugin hosts that own all device memory).  Fed the oracle's
schedule it must give the oracle's y, call after call, although its
accumulator is one fixed array shared by every call; it must also agree with
omni_expert_forward on the same schedule.  Its size limit is checked on the
CPU (tests/test_abi_cpu.py).  This file is collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
from atomic_expert_routing_b200 import _lib
import oracle as O
import workloads as WL
from helpers import dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu


def _oracle_case(cfg):
    """Seeded inputs, the oracle's routing and schedule (as device tensors) and
    the oracle's expert-centric y of that schedule."""
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    oi, og, _ = O.route(cfg, h)
    g32 = og.astype(np.float32)
    ref_s = O.schedule(cfg, oi, g32.astype(np.float64))
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    counts = torch.tensor([ref_s["n_active"], ref_s["n_groups"], 0, 0], dtype=torch.int32,
                          device="cuda")
    sched = {"task_token": dev(ref_s["task_token"]), "task_expert": dev(ref_s["task_expert"]),
             "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
             "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]), "counts": counts}
    return d, sched, y_ref


def _call_abi(D, d, sched, y):
    dd = D.c()
    return _lib.load().omni_expert_forward_noalloc(
        C.byref(dd), C.c_void_p(d["x"].data_ptr()), C.c_void_p(d["W"].data_ptr()),
        C.c_void_p(d["V"].data_ptr()), C.c_void_p(sched["task_token"].data_ptr()),
        C.c_void_p(sched["task_expert"].data_ptr()), C.c_void_p(sched["task_gate"].data_ptr()),
        C.c_void_p(sched["uniq"].data_ptr()), C.c_void_p(sched["group_off"].data_ptr()),
        C.c_void_p(sched["counts"].data_ptr()), C.c_void_p(y.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("cfg", [
    WL.Config("noalloc-bf16", L=96, d=256, Nr=32, Nc=48, k=8, K=8, B=16, dtype=WL.BF16, seed=21),
    WL.Config("noalloc-f32", L=40, d=64, Nr=16, Nc=16, k=6, K=6, B=8, dtype=WL.F32, seed=22),
    # the largest batch the array takes: L * d = 4 Mi
    WL.Config("noalloc-largest", L=2048, d=2048, Nr=32, Nc=32, k=4, K=4, B=16, dtype=WL.BF16,
              seed=23),
], ids=lambda c: c.name)
def test_noalloc_matches_oracle_twice(cfg):
    D = omni.LayerDims.of(cfg)
    d, sched, y_ref = _oracle_case(cfg)
    y_ws = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    # two calls in a row through the C ABI: the shared accumulator must be
    # cleared by every call (the second call sees the first call's sums)
    for _ in range(2):
        y = torch.full_like(y_ws, float("nan"))
        assert _call_abi(D, d, sched, y) == _lib.OMNI_OK
        torch.cuda.synchronize()
        yh = host_f64(y)
        assert rel_err(yh, y_ref) <= tol_y(cfg)
        assert rel_err(yh, host_f64(y_ws)) <= tol_y(cfg)
    assert int(sched["counts"][2].item()) == 0


def test_noalloc_binding_on_the_tensors_device():
    """The Python binding runs the call with the tensors' device current."""
    cfg = WL.Config("noalloc-dev", L=32, d=64, Nr=8, Nc=8, k=4, K=4, B=4, dtype=WL.BF16, seed=24)
    D = omni.LayerDims.of(cfg)
    d, sched, y_ref = _oracle_case(cfg)
    with torch.cuda.device(d["x"].device):
        y = omni.expert_forward_noalloc(D, d["x"], d["W"], d["V"], sched)
    torch.cuda.synchronize()
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
