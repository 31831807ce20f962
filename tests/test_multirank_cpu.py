"""Host logic of the data-parallel bench (one rank per GPU, no collective on
the data path) on two gloo ranks on the CPU: the step time is the slowest
rank's, the job throughput counts every rank's batch, and each rank gets its
own token batch with the shared weights."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as WL

CFG = WL.Config("ranks", L=16, d=64, Nr=8, Nc=8, k=2, K=2, B=4, dtype=WL.BF16, seed=5)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        x = bench.rank_inputs(CFG, rank)["x"]
        np.save(os.path.join(out_dir, f"x{rank}.npy"), x)
        with open(os.path.join(out_dir, f"ms{rank}.txt"), "w") as f:
            f.write(repr(ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_reduce_to_the_slowest(tmp_path):
    times = [1.25, 3.5]
    mp.spawn(_rank_main, args=(2, _free_port(), times, str(tmp_path)), nprocs=2, join=True)
    got = [float(open(tmp_path / f"ms{r}.txt").read()) for r in range(2)]
    assert got == [max(times)] * 2
    x0, x1 = np.load(tmp_path / "x0.npy"), np.load(tmp_path / "x1.npy")
    assert x0.shape == x1.shape == (CFG.L, CFG.d)
    assert not np.array_equal(x0, x1)  # each rank its own batch
    # rank 0's batch is the workload's own; other ranks' are seeded apart
    np.testing.assert_array_equal(x0, WL.make_inputs(CFG, experts=False)["x"])


def test_rank_inputs_share_the_router_weights():
    a, b = bench.rank_inputs(CFG, 0), bench.rank_inputs(CFG, 3)
    for key in ("Wr", "Wc"):
        np.testing.assert_array_equal(a[key], b[key])
    assert not np.array_equal(a["x"], b["x"])
    np.testing.assert_array_equal(b["x"], bench.rank_inputs(CFG, 3)["x"])  # deterministic


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1, 16384, 2.0) == pytest.approx(8.192e6)
    assert bench.job_throughput(4, 16384, 2.0) == pytest.approx(4 * 8.192e6)
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5


# ------------------------------------------------- expert-sharded forward (host logic)

SHARD_CFG = WL.Config("shards", L=24, d=64, Nr=8, Nc=8, k=4, K=4, B=3, dtype=WL.F32, seed=9)


def _shard_main(rank, world, port, out_dir):
    """One process of an expert-sharded forward with the oracle in place of
    the kernels: the whole batch's routing, this rank's experts only (other
    rows replaced by garbage that must not leak), the partials summed by
    sharded.combine over gloo."""
    import torch
    import oracle as O
    from atomic_expert_routing_b200 import sharded

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = SHARD_CFG
        h = WL.make_inputs(cfg)
        idx, gate, _ = O.route(cfg, h)
        lo, hi = sharded.shard_ranges(cfg.N, world)[rank]
        local = dict(h)
        for key in ("W", "V"):
            rows = np.full_like(h[key], 1e6)
            rows[lo:hi] = h[key][lo:hi]
            local[key] = rows
        inside = (idx >= lo) & (idx < hi)
        y_part, _ = O.forward_token(cfg, local, idx, np.where(inside, gate, 0.0))
        y = sharded.combine(torch.from_numpy(y_part.astype(np.float32)))
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_expert_shards_sum_to_the_layer(tmp_path, world):
    import oracle as O
    mp.spawn(_shard_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    h = WL.make_inputs(SHARD_CFG)
    idx, gate, _ = O.route(SHARD_CFG, h)
    y_ref, _ = O.forward_token(SHARD_CFG, h, idx, gate)
    for r in range(world):
        y = np.load(tmp_path / f"y{r}.npy")
        np.testing.assert_allclose(y, y_ref, rtol=1e-5, atol=1e-6 * np.abs(y_ref).max())


def test_shard_ranges_partition_the_ids():
    from atomic_expert_routing_b200 import sharded
    for N, G in ((1, 1), (7, 3), (64, 8), (1 << 20, 7), (10, 10)):
        r = sharded.shard_ranges(N, G)
        assert len(r) == G and r[0][0] == 0 and r[-1][1] == N
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        sizes = [hi - lo for lo, hi in r]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    for N, G in ((3, 4), (5, 0)):
        with pytest.raises(ValueError):
            sharded.shard_ranges(N, G)


def _gather_main(rank, world, port, L, K, out_dir):
    """Each rank holds the routing of its token_ranges share (ids and gates
    that encode the token and slot); gather_routing assembles the batch."""
    import torch
    from atomic_expert_routing_b200 import sharded

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t0, t1 = sharded.token_ranges(L, world)[rank]
        tok = torch.arange(t0, t1, dtype=torch.int32)[:, None]
        slot = torch.arange(K, dtype=torch.int32)[None, :]
        idx = (tok * 1000 + slot).contiguous()
        gate = (tok.float() + slot.float() / 100.0).contiguous()
        gi, gg = sharded.gather_routing(idx, gate, L)
        np.save(os.path.join(out_dir, f"gi{rank}.npy"), gi.numpy())
        np.save(os.path.join(out_dir, f"gg{rank}.npy"), gg.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,L", [(2, 10), (3, 7), (3, 2)])
def test_routing_shares_gather_to_the_batch(tmp_path, world, L):
    K = 4
    mp.spawn(_gather_main, args=(world, _free_port(), L, K, str(tmp_path)), nprocs=world,
             join=True)
    want_i = np.arange(L)[:, None] * 1000 + np.arange(K)[None, :]
    want_g = (np.arange(L)[:, None] + np.arange(K)[None, :] / 100.0).astype(np.float32)
    for r in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"gi{r}.npy"), want_i)
        np.testing.assert_array_equal(np.load(tmp_path / f"gg{r}.npy"), want_g)


def test_token_ranges_cover_the_batch():
    from atomic_expert_routing_b200 import sharded
    for L, G in ((10, 3), (7, 7), (2, 3), (0, 2), (16384, 8)):
        r = sharded.token_ranges(L, G)
        assert len(r) == G and r[0][0] == 0 and r[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
