"""GPU parity of the expert-sharded forward (omni_moe_forward_shard): every
shard of a partition of the ids runs on this GPU in turn, as the processes of
a group would, and is checked on its own and in sum.

Per shard: the routing equals the unsharded forward's bit for bit; the fp32
partial y equals the oracle's token-centric y of the same routing with the
gates of other shards' experts set to zero (max|dy| / max|y| <= 1e-4: fp32
accumulation of bf16-exact inputs, no output rounding); counts[0], counts[1]
are the shard's active ids and their groups.  In sum: the partials, added
and cast, match the oracle's y of the whole layer at the storage bar.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import atomic_expert_routing_b200.sharded as sharded
import oracle as O
import workloads as WL
from helpers import dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu

CONFIGS = [
    # the routing-order tail (decode shape)
    WL.Config("shard-tail-bf16-d2048", L=64, d=2048, Nr=128, Nc=128, k=64, K=64, B=128,
              dtype=WL.BF16, seed=81),
    WL.Config("shard-tail-f32-d256", L=40, d=256, Nr=32, Nc=48, k=8, K=8, B=16, dtype=WL.F32,
              seed=82),
    # routing -> schedule -> grouped execution
    WL.Config("shard-staged-bf16-d512", L=2048, d=512, Nr=128, Nc=128, k=16, K=16, B=64,
              dtype=WL.BF16, seed=83),
    WL.Config("shard-ragged-bf16", L=130, d=72, Nr=48, Nc=80, k=7, K=5, B=4, dtype=WL.BF16,
              seed=84),
    # column-slice sweeps over the window order
    WL.Config("shard-sweeps-bf16", L=8192, d=2048, Nr=64, Nc=64, k=8, K=8, B=32, dtype=WL.BF16,
              seed=85),
    WL.Config("shard-sweeps-f32", L=12288, d=1024, Nr=48, Nc=40, k=6, K=5, B=16, dtype=WL.F32,
              seed=86),
]
PART_TOL = 1e-4


def _inputs(cfg, gated=False):
    h = WL.make_inputs(cfg)
    if gated:
        h.update(WL.make_gate(cfg))
    return h, {k: dev(v) for k, v in h.items()}


def _unsharded(cfg, d, U=None):
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         U=U, idx=idx, gate=gate)
    torch.cuda.synchronize()
    return y, idx.cpu().numpy(), gate.cpu().numpy()


def _run_shards(cfg, h, d, G, gated=False, flags=0, routed=False):
    """Every shard of the G-way split in turn; returns the summed partials.
    routed: the shards take the unsharded call's routing as input
    (omni_moe_forward_shard_routed) instead of routing the batch."""
    D = omni.LayerDims.of(cfg, flags=flags)
    U = d.get("U") if gated else None
    y_full, i_ref, g_ref = _unsharded(cfg, d, U)
    i_dev, g_dev = torch.from_numpy(i_ref).cuda(), torch.from_numpy(g_ref).cuda()
    total = torch.zeros((cfg.L, cfg.d), dtype=torch.float32, device="cuda")
    active = np.unique(i_ref)
    for lo, hi in sharded.shard_ranges(cfg.N, G):
        idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
        gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
        counts = omni.new_counts("cuda")
        if routed:
            yp = omni.moe_forward_shard_routed(D, d["x"], d["W"][lo:hi], d["V"][lo:hi], lo, hi,
                                               i_dev, g_dev,
                                               U=U[lo:hi] if U is not None else None,
                                               counts=counts)
            idx.copy_(i_dev)
            gate.copy_(g_dev)
        else:
            yp = omni.moe_forward_shard(D, d["x"], d["Wr"], d["Wc"], d["W"][lo:hi],
                                        d["V"][lo:hi], lo, hi, d["bias_r"], d["bias_c"],
                                        U=U[lo:hi] if U is not None else None, counts=counts,
                                        idx=idx, gate=gate)
        torch.cuda.synchronize()
        gi, gg, c = idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy()
        assert np.array_equal(gi, i_ref) and np.array_equal(gg, g_ref)
        assert c[2] == 0
        mine = int(np.count_nonzero((active >= lo) & (active < hi)))
        assert c[0] == mine and c[1] == (mine + cfg.B - 1) // cfg.B
        # the oracle's partial: the same routing, other shards' gates zeroed
        inside = (gi >= lo) & (gi < hi)
        y_ref, _ = O.forward_token(cfg, h, gi, np.where(inside, gg, 0.0).astype(np.float64))
        yp_h = host_f64(yp)
        if not inside.any():
            assert not yp_h.any()
        else:
            assert rel_err(yp_h, y_ref) <= PART_TOL
            assert not yp_h[~inside.any(axis=1)].any()  # tokens without a task here: 0
        total += yp
    y = omni.cast_output(D, total)
    y_ref, _ = O.forward_token(cfg, h, i_ref, g_ref.astype(np.float64))
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
    assert rel_err(host_f64(y), host_f64(y_full)) <= tol_y(cfg)


@pytest.mark.parametrize("G", [1, 2, 3, 8])
@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_shards_partition_the_layer(cfg, G):
    h, d = _inputs(cfg)
    _run_shards(cfg, h, d, G)


@pytest.mark.parametrize("cfg", CONFIGS[2:], ids=lambda c: c.name)
def test_shards_on_the_scheduled_paths(cfg):
    """OMNI_FLAG_STAGED_SMALL keeps batches whose rows fit in L2 on the
    schedule-based paths (grouped kernels, or the window order of the
    sweeps), which the shard's task range bounds."""
    h, d = _inputs(cfg)
    _run_shards(cfg, h, d, 3, flags=omni.OMNI_FLAG_STAGED_SMALL)


@pytest.mark.parametrize("flags", [0, omni.OMNI_FLAG_STAGED_SMALL], ids=["default", "scheduled"])
@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_shards_from_a_given_routing(cfg, flags):
    """omni_moe_forward_shard_routed: the shards take the batch's routing as
    input (as the processes of a group do after exchanging their shares of
    it) and give the same partials."""
    h, d = _inputs(cfg)
    _run_shards(cfg, h, d, 3, flags=flags, routed=True)


@pytest.mark.parametrize("cfg", [CONFIGS[0], CONFIGS[2], CONFIGS[4]], ids=lambda c: c.name)
def test_gated_shards(cfg):
    h, d = _inputs(cfg, gated=True)
    _run_shards(cfg, h, d, 3, gated=True)


def test_a_shard_without_active_ids_writes_zeros():
    """Ids no token selects: the partial is exactly zero and the counts 0."""
    cfg = WL.Config("shard-idle", L=16, d=256, Nr=64, Nc=64, k=2, K=2, B=8, dtype=WL.BF16,
                    seed=87)
    h, d = _inputs(cfg)
    _, i_ref, _ = _unsharded(cfg, d)
    free = np.setdiff1d(np.arange(cfg.N), i_ref)
    lo = int(free[0])
    hi = lo + 1
    D = omni.LayerDims.of(cfg)
    counts = omni.new_counts("cuda")
    yp = torch.full((cfg.L, cfg.d), 7.0, dtype=torch.float32, device="cuda")
    omni.moe_forward_shard(D, d["x"], d["Wr"], d["Wc"], d["W"][lo:hi], d["V"][lo:hi], lo, hi,
                           d["bias_r"], d["bias_c"], y_part=yp, counts=counts)
    torch.cuda.synchronize()
    assert not yp.any()
    assert counts[0].item() == 0 and counts[1].item() == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("split_routing", [False, True], ids=["replicated", "split-routing"])
def test_sharded_forward_over_a_one_process_nccl_group(split_routing):
    """sharded.forward (and forward_split_routing, whose all-gathers are then
    trivial) end to end, the all-reduce on NCCL, in a group of one process
    holding every id: y as the unsharded forward's, within the storage bar
    of the oracle."""
    import torch.distributed as dist
    cfg = CONFIGS[2]
    h, d = _inputs(cfg)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        D = omni.LayerDims.of(cfg)
        fwd = sharded.forward_split_routing if split_routing else sharded.forward
        y = fwd(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], 0, cfg.N, d["bias_r"], d["bias_c"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_full, gi, gg = _unsharded(cfg, d)
    y_ref, _ = O.forward_token(cfg, h, gi, gg.astype(np.float64))
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
    assert rel_err(host_f64(y), host_f64(y_full)) <= tol_y(cfg)
