"""GPU parity of gated (SwiGLU) atomic experts, h = SiLU(x.W[e]) * (x.U[e]),
against the fp64 oracle, on every execution path that takes U: the
small-batch tail of the fused forward and the staged kernels it replaces,
the staged grouped execution (per-group and accumulator kernels), the
column-slice sweeps (staged and fused), and the token-centric ablation.

Bars as for the plain expert: max|dy| / max|y| <= 1e-4 (fp32 storage) or
2e-2 (bf16 storage, fp32 accumulation); |U| and the group count exact.
"""
import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from helpers import dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu

# the routing-order tail (one config per row width it compiles for, both
# storage types, a ragged batch and a skewed one)
TAIL = [
    WL.Config("glu-tail-bf16-d256", L=1, d=256, Nr=16, Nc=16, k=4, K=4, B=200, dtype=WL.BF16,
              seed=61),
    WL.Config("glu-tail-bf16-d512", L=37, d=512, Nr=40, Nc=30, k=16, K=16, B=7, dtype=WL.BF16,
              seed=62),
    WL.Config("glu-tail-bf16-d1024-skew", L=100, d=1024, Nr=64, Nc=64, k=8, K=8, B=64,
              dtype=WL.BF16, seed=63, zipf_s=1.1),
    WL.Config("glu-tail-bf16-d2048-decode", L=64, d=2048, Nr=128, Nc=128, k=64, K=64, B=128,
              dtype=WL.BF16, seed=64),
    WL.Config("glu-tail-f32-d128", L=50, d=128, Nr=32, Nc=32, k=6, K=6, B=16, dtype=WL.F32,
              seed=65),
    WL.Config("glu-tail-f32-d1024", L=20, d=1024, Nr=16, Nc=16, k=4, K=4, B=5, dtype=WL.F32,
              seed=66),
]
# batches above the tail's size: routing -> schedule -> grouped execution
STAGED = [
    WL.TINY.with_(name="glu-tiny-fp32", seed=67),
    WL.Config("glu-bf16-d512", L=2048, d=512, Nr=128, Nc=128, k=16, K=16, B=64, dtype=WL.BF16,
              seed=68),
    WL.Config("glu-bf16-d2048", L=2048, d=2048, Nr=128, Nc=128, k=32, K=32, B=128,
              dtype=WL.BF16, seed=69),
    WL.Config("glu-ragged-bf16", L=130, d=72, Nr=48, Nc=80, k=7, K=5, B=4, dtype=WL.BF16,
              seed=70),
    WL.Config("glu-ragged-f32", L=37, d=40, Nr=12, Nc=20, k=9, K=9, B=2, dtype=WL.F32, seed=71),
]
# fp32 accumulators above ~40 MiB: column-slice sweeps
SWEEP = [
    WL.Config("glu-sweeps-bf16", L=8192, d=2048, Nr=64, Nc=64, k=8, K=8, B=32, dtype=WL.BF16,
              seed=72),
    WL.Config("glu-sweeps-f32", L=12288, d=1024, Nr=48, Nc=40, k=6, K=5, B=16, dtype=WL.F32,
              seed=73),
]


def _inputs(cfg):
    h = dict(WL.make_inputs(cfg), **WL.make_gate(cfg))
    return h, {k: dev(v) for k, v in h.items()}


def _fused(cfg, d, flags=0):
    D = omni.LayerDims.of(cfg, flags=flags)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         U=d["U"], counts=counts, idx=idx, gate=gate)
    torch.cuda.synchronize()
    return y, idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy()


def _check_fused(cfg, h, y, gi, gg, c):
    """y against the oracle's gated expert-centric y of the routing the GPU
    chose (routing parity itself is the plain tests' subject), |U| and the
    group count exactly."""
    ref_s = O.schedule(cfg, gi, gg.astype(np.float64))
    assert c[2] == 0
    assert c[0] == ref_s["n_active"] and c[1] == ref_s["n_groups"]
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    err = rel_err(host_f64(y), y_ref)
    assert err <= tol_y(cfg), err
    return y_ref


def _oracle_schedule(cfg, h):
    oi, og, _ = O.route(cfg, h)
    g32 = og.astype(np.float32)
    ref_s = O.schedule(cfg, oi, g32.astype(np.float64))
    counts = torch.tensor([ref_s["n_active"], ref_s["n_groups"], 0, 0], dtype=torch.int32,
                          device="cuda")
    sched = {"task_token": dev(ref_s["task_token"]), "task_expert": dev(ref_s["task_expert"]),
             "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
             "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]), "counts": counts}
    return oi, g32, ref_s, sched


@pytest.mark.parametrize("cfg", TAIL, ids=lambda c: c.name)
def test_gated_small_batch_tail(cfg):
    """The two-kernel tail with U, and the scheduled kernels
    (OMNI_FLAG_STAGED_SMALL) on the same routing."""
    h, d = _inputs(cfg)
    y1, i1, g1, c1 = _fused(cfg, d)
    y2, i2, g2, c2 = _fused(cfg, d, omni.OMNI_FLAG_STAGED_SMALL)
    assert np.array_equal(i1, i2) and np.array_equal(g1, g2)
    _check_fused(cfg, h, y1, i1, g1, c1)
    _check_fused(cfg, h, y2, i2, g2, c2)


@pytest.mark.parametrize("cfg", STAGED, ids=lambda c: c.name)
def test_gated_expert_forward_from_oracle_schedule(cfg):
    h, d = _inputs(cfg)
    _, _, ref_s, sched = _oracle_schedule(cfg, h)
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    y = omni.expert_forward(omni.LayerDims.of(cfg), d["x"], d["W"], d["V"], sched, U=d["U"])
    err = rel_err(host_f64(y), y_ref)
    assert err <= tol_y(cfg), err
    assert int(sched["counts"][2].item()) == 0


@pytest.mark.parametrize("cfg", STAGED, ids=lambda c: c.name)
def test_gated_fused_forward(cfg):
    h, d = _inputs(cfg)
    y, gi, gg, c = _fused(cfg, d)
    _check_fused(cfg, h, y, gi, gg, c)


@pytest.mark.parametrize("cfg", STAGED[:3], ids=lambda c: c.name)
def test_gated_token_centric(cfg):
    h, d = _inputs(cfg)
    oi, g32, _, _ = _oracle_schedule(cfg, h)
    y_ref, _ = O.forward_token(cfg, h, oi, g32.astype(np.float64))
    y = omni.token_centric_forward(omni.LayerDims.of(cfg), d["x"], d["W"], d["V"], dev(oi),
                                   dev(g32), U=d["U"])
    err = rel_err(host_f64(y), y_ref)
    assert err <= tol_y(cfg), err


@pytest.mark.parametrize("cfg", SWEEP, ids=lambda c: c.name)
def test_gated_sweeps(cfg):
    """Staged sweeps from the oracle's schedule, and the fused forward's
    window order, both with U."""
    assert cfg.L * cfg.d * 4 > (40 << 20)
    h, d = _inputs(cfg)
    _, _, ref_s, sched = _oracle_schedule(cfg, h)
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    y = omni.expert_forward(omni.LayerDims.of(cfg), d["x"], d["W"], d["V"], sched, U=d["U"])
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
    # the fused forward on the window path (the default takes the tail: the
    # batch's rows fit in L2) and by default
    for flags in (omni.OMNI_FLAG_STAGED_SMALL, 0):
        y, gi, gg, c = _fused(cfg, d, flags)
        _check_fused(cfg, h, y, gi, gg, c)


def test_gated_ignores_the_dense_tensor_core_flag():
    """OMNI_FLAG_DENSE_TENSOR_CORES computes plain activations only; with U
    the groups run on the CUDA-core kernels and y still matches the oracle."""
    cfg = WL.Config("glu-dense-groups", L=8192, d=1024, Nr=16, Nc=16, k=8, K=8, B=128,
                    dtype=WL.BF16, seed=74)
    h, d = _inputs(cfg)
    _, _, ref_s, sched = _oracle_schedule(cfg, h)
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    D = omni.LayerDims.of(cfg, flags=omni.OMNI_FLAG_DENSE_TENSOR_CORES)
    y = omni.expert_forward(D, d["x"], d["W"], d["V"], sched, U=d["U"])
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
    assert int(sched["counts"][3].item()) == 0  # no dense group was planned


def test_gate_matrix_changes_the_output():
    """U reaches the kernels: the gated y of a batch differs from the plain y
    of the same batch by far more than rounding (the gated form's reduction
    to the plain one is pinned on the oracle)."""
    cfg = TAIL[2]
    h, d = _inputs(cfg)
    y_glu, i1, g1, _ = _fused(cfg, d)
    D = omni.LayerDims.of(cfg)
    y_plain = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"],
                               d["bias_c"])
    assert rel_err(host_f64(y_glu), host_f64(y_plain)) > 0.1
