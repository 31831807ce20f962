"""GPU parity of the tensor-core activations of dense groups
(OMNI_FLAG_DENSE_TENSOR_CORES; off by default).

Groups whose tasks average at least 384 per touched block of 128 tokens have
their activations c = gate * SiLU(x[t] . W[e]) formed as entries of the dense
products X[block] W_g^T on the tensor cores (tcgen05); the grouped-execution
kernel adds c * V[e] for them and forms the rest itself.  counts[3] reports
how many groups took the tensor cores (at most 64 per call), so each case
checks the path it means to test, and y is compared with the oracle's
expert-centric execution of the same schedule.  Bar: max|dy| / max|y| <= 2e-2
(bf16 storage, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from helpers import dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu


TC = omni.OMNI_FLAG_DENSE_TENSOR_CORES


def _run(cfg, idx, gate, inputs=None, flags=TC):
    """Grouped execution of the oracle's schedule of (idx, gate): the GPU's y
    and counts, and the oracle's y."""
    h = inputs if inputs is not None else WL.make_inputs(cfg)
    g32 = gate.astype(np.float32)
    ref_s = O.schedule(cfg, idx, g32.astype(np.float64))
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    counts = torch.tensor([ref_s["n_active"], ref_s["n_groups"], 0, -1], dtype=torch.int32,
                          device="cuda")
    sched = {"task_token": dev(ref_s["task_token"]), "task_expert": dev(ref_s["task_expert"]),
             "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
             "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]), "counts": counts}
    d = {k: dev(h[k]) for k in ("x", "W", "V")}
    D = omni.LayerDims.of(cfg, flags=flags)
    y = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    return host_f64(y), counts.cpu().numpy(), y_ref, ref_s


def _pool_routing(cfg, pool, seed):
    """Every token takes K distinct experts from one pool of ids: the groups
    of the pool's experts are dense."""
    rng = np.random.default_rng(seed)
    ids = np.sort(rng.choice(cfg.N, size=pool, replace=False))
    idx = np.stack([rng.choice(ids, size=cfg.K, replace=False) for _ in range(cfg.L)])
    gate = (1.0 - rng.random((cfg.L, cfg.K))).astype(np.float32)
    return idx.astype(np.int32), gate


@pytest.mark.parametrize("cfg,pool,want", [
    # two groups of 128 (128-wide panels), 512 tasks per touched tile
    (WL.Config("dense-128", L=2048, d=512, Nr=16, Nc=16, k=8, K=8, B=128, dtype=WL.BF16,
               seed=71), 256, 2),
    # four groups, d = 1024, a ragged last token block
    (WL.Config("dense-d1024-ragged", L=1000, d=1024, Nr=32, Nc=32, k=16, K=16, B=128,
               dtype=WL.BF16, seed=72), 512, 4),
    # 80 dense groups of 16: 64 take the tensor cores, 16 the CUDA cores
    (WL.Config("dense-over-cap", L=1024, d=256, Nr=256, Nc=256, k=256, K=256, B=16,
               dtype=WL.BF16, seed=73), 1280, 64),
], ids=lambda c: c.name if hasattr(c, "name") else None)
def test_dense_groups_on_tensor_cores(cfg, pool, want):
    idx, gate = _pool_routing(cfg, pool, cfg.seed)
    y, counts, y_ref, _ = _run(cfg, idx, gate)
    assert counts[2] == 0
    assert counts[3] == want
    assert rel_err(y, y_ref) <= tol_y(cfg)


def test_sparse_groups_stay_on_cuda_cores():
    """Nearly distinct experts per task (a few tasks per tile): no group is
    dense, counts[3] = 0, y as the oracle's."""
    cfg = WL.Config("sparse", L=512, d=256, Nr=128, Nc=128, k=8, K=8, B=64, dtype=WL.BF16, seed=74)
    idx, gate = WL.random_routing(cfg, pool=cfg.N)
    y, counts, y_ref, _ = _run(cfg, idx, gate)
    assert counts[2] == 0 and counts[3] == 0
    assert rel_err(y, y_ref) <= tol_y(cfg)


def test_skewed_workload_mixes_both_paths():
    """The Zipf-skewed workload's routing on a sub-batch: some groups dense,
    some not; y as the oracle's."""
    cfg = WL.SKEWED
    tok = WL.sample_tokens(cfg, 2048)
    h = WL.make_inputs(cfg)
    cs = cfg.with_(L=len(tok))
    hs = dict(h, x=np.ascontiguousarray(h["x"][tok]))
    oi, og, _ = O.route(cs, hs)
    y, counts, y_ref, ref_s = _run(cs, oi, og.astype(np.float32), inputs=hs)
    assert counts[2] == 0
    assert 0 < counts[3] < ref_s["n_groups"] or counts[3] == min(64, ref_s["n_groups"])
    assert rel_err(y, y_ref) <= tol_y(cs)


def test_wide_groups_stay_on_cuda_cores():
    """Groups of more than 128 experts are not formed on the tensor cores
    (the tile holds 128 experts): counts[3] is left as the caller set it."""
    cfg = WL.Config("wide-groups", L=1024, d=256, Nr=32, Nc=32, k=8, K=8, B=256, dtype=WL.BF16,
                    seed=75)
    idx, gate = _pool_routing(cfg, 512, cfg.seed)
    y, counts, y_ref, _ = _run(cfg, idx, gate)
    assert counts[2] == 0 and counts[3] == -1
    assert rel_err(y, y_ref) <= tol_y(cfg)


def test_dense_path_is_off_without_the_flag():
    cfg = WL.Config("dense-off", L=2048, d=512, Nr=16, Nc=16, k=8, K=8, B=128, dtype=WL.BF16,
                    seed=76)
    idx, gate = _pool_routing(cfg, 256, cfg.seed)
    y, counts, y_ref, _ = _run(cfg, idx, gate, flags=0)
    assert counts[2] == 0 and counts[3] == -1
    assert rel_err(y, y_ref) <= tol_y(cfg)
