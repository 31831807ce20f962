"""omni_expert_forward_noalloc: the grouped execution for callers that cannot
allocate device memory while the layer runs (graph capture, ahead-of-time
memory plans, plugin hosts that own all device memory).  It must give the same
y as omni_expert_forward, call after call, although its accumulator is one
fixed array shared by every call.  This file is collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
from atomic_expert_routing_b200 import _lib
import workloads as WL
from helpers import dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu


def _case(cfg):
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx, gate, _ = omni.route(D, d["x"], d["Wr"], d["Wc"], d["bias_r"], d["bias_c"])
    sched = omni.schedule(D, idx, gate)
    return D, d, sched


@pytest.mark.parametrize("cfg", [
    WL.Config("noalloc-bf16", L=96, d=256, Nr=32, Nc=48, k=8, K=8, B=16, dtype=WL.BF16, seed=21),
    WL.Config("noalloc-f32", L=40, d=64, Nr=16, Nc=16, k=4, K=6, B=8, dtype=WL.F32, seed=22),
    # the largest batch the array takes: L * d = 4 Mi, with the per-token counts behind it
    WL.Config("noalloc-largest", L=2048, d=2048, Nr=32, Nc=32, k=4, K=4, B=16, dtype=WL.BF16,
              seed=23),
], ids=lambda c: c.name)
def test_noalloc_matches_workspace_path_twice(cfg):
    D, d, sched = _case(cfg)
    y_ref = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    # two calls in a row through the C ABI: the shared accumulator must be
    # cleared by every call
    for _ in range(2):
        y = torch.full_like(y_ref, float("nan"))
        dd = D.c()
        rc = _lib.load().omni_expert_forward_noalloc(
            C.byref(dd), C.c_void_p(d["x"].data_ptr()), C.c_void_p(d["W"].data_ptr()),
            C.c_void_p(d["V"].data_ptr()), C.c_void_p(sched["task_token"].data_ptr()),
            C.c_void_p(sched["task_expert"].data_ptr()), C.c_void_p(sched["task_gate"].data_ptr()),
            C.c_void_p(sched["uniq"].data_ptr()), C.c_void_p(sched["group_off"].data_ptr()),
            C.c_void_p(sched["counts"].data_ptr()), C.c_void_p(y.data_ptr()),
            C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == _lib.OMNI_OK
        torch.cuda.synchronize()
        assert rel_err(host_f64(y), host_f64(y_ref)) <= tol_y(cfg)
    assert int(sched["counts"][2].item()) == 0


def test_noalloc_rejects_batches_beyond_its_array():
    cfg = WL.Config("noalloc-big", L=4096, d=2048, Nr=32, Nc=32, k=4, K=4, B=16, dtype=WL.BF16)
    D = omni.LayerDims.of(cfg)  # L * d = 8 Mi > 4 Mi floats
    fake = C.c_void_p(4096)
    dd = D.c()
    rc = _lib.load().omni_expert_forward_noalloc(C.byref(dd), *([fake] * 10), None)
    assert rc == _lib.OMNI_ERR_UNSUPPORTED
