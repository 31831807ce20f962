"""GPU parity: every stage of the CUDA path against the fp64 oracle.

Each stage is fed the oracle's own inputs (logits, routing, schedule) so errors
do not compound; the fused call is then compared end to end.  Large
configurations run the oracle on a seeded sub-batch of tokens (rows of x; the
layer is row-independent) and, at full size, check sampled rows plus
properties that hold at any size.

Bars: integer outputs bit-exact (selected ids except reported near-ties, the
task permutation, unique ids, group boundaries); y within
max|dy| / max|y| <= 1e-4 (fp32 storage) or 2e-2 (bf16 storage, fp32
accumulation); gates/scores within fp32 rounding of the oracle.
"""
import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from helpers import check_selection, dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu

ALL = [WL.TINY, WL.BF16_16K, WL.SKEWED, WL.PREFILL, WL.DECODE]
IDS = [c.name for c in ALL]
SUB = {WL.TINY.name: 128, WL.BF16_16K.name: 4096, WL.SKEWED.name: 1024,
       WL.PREFILL.name: 512, WL.DECODE.name: 64}

_HOST_R, _HOST_E, _DEV_R, _DEV_E = {}, {}, {}, {}


def _keys(cfg):
    return ((cfg.seed, cfg.L, cfg.d, cfg.Nr, cfg.Nc, cfg.dtype, cfg.zipf_s),
            (cfg.seed, cfg.Nr, cfg.Nc, cfg.d, cfg.dtype))


def host_inputs(cfg):
    """Seeded inputs, cached for the session (experts shared by configs with equal N, d)."""
    kr, ke = _keys(cfg)
    if kr not in _HOST_R:
        _HOST_R[kr] = WL.make_inputs(cfg, experts=False)
    if ke not in _HOST_E:
        _HOST_E[ke] = WL.make_experts(cfg)
    return dict(_HOST_R[kr], **_HOST_E[ke])


def dev_inputs(cfg):
    kr, ke = _keys(cfg)
    h = host_inputs(cfg)
    if kr not in _DEV_R:
        _DEV_R[kr] = {k: dev(h[k]) for k in ("x", "Wr", "Wc", "bias_r", "bias_c")}
    if ke not in _DEV_E:
        _DEV_E[ke] = {k: dev(h[k]) for k in ("W", "V")}
    return dict(_DEV_R[kr], **_DEV_E[ke])


def sub_batch(cfg, n=None):
    """A seeded sub-batch of tokens as its own batch: (cfg_s, host inputs, device inputs)."""
    n = SUB[cfg.name] if n is None else n
    h = host_inputs(cfg)
    d = dev_inputs(cfg)
    if n >= cfg.L:
        return cfg, h, d
    tok = WL.sample_tokens(cfg, n)
    hs = dict(h, x=np.ascontiguousarray(h["x"][tok]))
    ds = dict(d, x=d["x"][torch.from_numpy(tok).to(d["x"].device)].contiguous())
    return cfg.with_(L=n), hs, ds


def oracle_route_full(cfg, h):
    lr, lc = O.axis_logprobs(cfg, h)
    idx, gate, score = O.select(cfg, lr, lc)
    bi, bg, bs, nxt = O.select_bruteforce(cfg, lr, lc)
    assert np.array_equal(idx, bi)
    return idx, gate, score, nxt, lr, lc


# --------------------------------------------------------------------------- router


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_router_logits(cfg):
    """Router projections (tcgen05 for bf16, CUDA cores for fp32) vs the oracle's
    fp64 logits; error bound: fp32 accumulation of d exact products,
    |dz| <= 2 d 2^-24 sum|x_m w_m|."""
    cs, h, d = sub_batch(cfg, min(SUB[cfg.name], 512))
    D = omni.LayerDims.of(cs)
    z = omni.router_logits(D, d["x"], d["Wr"], d["Wc"]).cpu().numpy().astype(np.float64)
    hb = dict(h, bias_r=None, bias_c=None)
    zr, zc = O.axis_logits(cs, hb)
    ref = np.concatenate([zr, zc], axis=1)
    f = (lambda a: WL.bf16_bits_to_f32(a)) if cs.dtype == WL.BF16 else (lambda a: a)
    xa = np.abs(f(h["x"]).astype(np.float64))
    wa = np.abs(np.concatenate([f(h["Wr"]), f(h["Wc"])]).astype(np.float64))
    bound = 2 * cs.d * 2.0 ** -24 * (xa @ wa.T) + 1e-30
    err = np.abs(z - ref)
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3g}"
    assert np.median(err / bound) < 0.05


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_route_select_from_oracle_logits(cfg):
    """Selection kernel alone: fed the oracle's logits rounded to fp32; compared
    with the oracle's selection from the same fp32 logits."""
    cs, h, _ = sub_batch(cfg)
    zr, zc = O.axis_logits(cs, h)  # biases included
    z32 = np.concatenate([zr, zc], axis=1).astype(np.float32)
    D = omni.LayerDims.of(cs)
    idx, gate, score = omni.route_select(D, dev(z32))
    lr = O.log_softmax(z32[:, :cs.Nr].astype(np.float64))
    lc = O.log_softmax(z32[:, cs.Nr:].astype(np.float64))
    oi, og, os_ = O.select(cs, lr, lc)
    _, _, bs, nxt = O.select_bruteforce(cs, lr, lc)
    ne, nn = check_selection(cs, idx.cpu().numpy(), gate.cpu().numpy(), score.cpu().numpy(),
                             oi, og, os_, nxt, lr, lc)
    assert ne > 0.7 * cs.L


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_route_end_to_end(cfg):
    cs, h, d = sub_batch(cfg)
    D = omni.LayerDims.of(cs)
    idx, gate, score = omni.route(D, d["x"], d["Wr"], d["Wc"], d["bias_r"], d["bias_c"])
    oi, og, os_, nxt, lr, lc = oracle_route_full(cs, h)
    ne, nn = check_selection(cs, idx.cpu().numpy(), gate.cpu().numpy(), score.cpu().numpy(),
                             oi, og, os_, nxt, lr, lc)
    assert ne > 0.7 * cs.L


def test_route_simt_diagnostic_path_matches_tensor_cores():
    cfg = WL.BF16_16K
    cs, h, d = sub_batch(cfg, 1024)
    D = omni.LayerDims.of(cs)
    Ds = omni.LayerDims.of(cs, flags=omni.OMNI_FLAG_ROUTER_SIMT)
    z_tc = omni.router_logits(D, d["x"], d["Wr"], d["Wc"])
    z_simt = omni.router_logits(Ds, d["x"], d["Wr"], d["Wc"])
    assert torch.allclose(z_tc, z_simt, rtol=0, atol=1e-4)
    oi, og, os_, nxt, lr, lc = oracle_route_full(cs, h)
    idx, gate, score = omni.route(Ds, d["x"], d["Wr"], d["Wc"])
    check_selection(cs, idx.cpu().numpy(), gate.cpu().numpy(), score.cpu().numpy(), oi, og, os_,
                    nxt, lr, lc)


# --------------------------------------------------------------------------- schedule


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_schedule_from_oracle_routing(cfg):
    """Scheduler fed the oracle's routing: bit-exact task order, unique ids,
    group boundaries and counts."""
    cs, h, _ = sub_batch(cfg, min(cfg.L, 2048))
    oi, og, _ = O.route(cs, h)
    g32 = og.astype(np.float32)
    ref = O.schedule(cs, oi, g32.astype(np.float64))
    D = omni.LayerDims.of(cs)
    s = omni.schedule(D, dev(oi), dev(g32))
    cnt = s["counts"].cpu().numpy()
    assert cnt[0] == ref["n_active"] and cnt[1] == ref["n_groups"] and cnt[2] == 0
    np.testing.assert_array_equal(s["task_token"].cpu().numpy(), ref["task_token"])
    np.testing.assert_array_equal(s["task_expert"].cpu().numpy(), ref["task_expert"])
    np.testing.assert_array_equal(s["task_gate"].cpu().numpy(), ref["task_gate"].astype(np.float32))
    np.testing.assert_array_equal(s["uniq"].cpu().numpy()[:cnt[0]], ref["uniq"])
    np.testing.assert_array_equal(s["group_off"].cpu().numpy()[:cnt[1] + 1], ref["group_off"])


@pytest.mark.parametrize("B", [1, 3, 10 ** 6])
def test_schedule_group_size_extremes(B):
    cfg = WL.TINY.with_(B=B)
    h = host_inputs(WL.TINY)
    oi, og, _ = O.route(cfg, h)
    g32 = og.astype(np.float32)
    ref = O.schedule(cfg, oi, g32.astype(np.float64))
    s = omni.schedule(omni.LayerDims.of(cfg), dev(oi), dev(g32))
    cnt = s["counts"].cpu().numpy()
    assert cnt[1] == ref["n_groups"]
    np.testing.assert_array_equal(s["task_expert"].cpu().numpy(), ref["task_expert"])
    np.testing.assert_array_equal(s["task_token"].cpu().numpy(), ref["task_token"])
    np.testing.assert_array_equal(s["group_off"].cpu().numpy()[:cnt[1] + 1], ref["group_off"])


SCHED = [
    # one cluster over a bitmap of all ids; K rounded up to a power of two
    # gives the segment each token's ids are sorted in
    WL.Config("bits-K1", L=500, d=8, Nr=32, Nc=64, k=1, K=1, B=100, dtype=WL.F32),
    WL.Config("bits-K3", L=37, d=8, Nr=12, Nc=20, k=3, K=3, B=2, dtype=WL.F32),
    WL.Config("bits-K16", L=256, d=8, Nr=256, Nc=256, k=16, K=16, B=64, dtype=WL.F32),
    WL.Config("bits-K32", L=100, d=8, Nr=512, Nc=512, k=32, K=32, B=50, dtype=WL.F32),
    WL.Config("bits-K64-M8192", L=128, d=8, Nr=1024, Nc=1024, k=64, K=64, B=128, dtype=WL.F32),
    WL.Config("bits-K100", L=20, d=8, Nr=64, Nc=64, k=64, K=100, B=7, dtype=WL.F32),
    WL.Config("bits-K256", L=16, d=8, Nr=128, Nc=64, k=64, K=256, B=64, dtype=WL.F32),
    WL.Config("bits-N4M", L=64, d=8, Nr=2048, Nc=2048, k=64, K=64, B=128, dtype=WL.F32),
    # the radix cluster sort: more than 2^22 ids, or more than 512 tokens
    WL.Config("cluster-N16M", L=64, d=8, Nr=4096, Nc=4096, k=64, K=64, B=128, dtype=WL.F32),
    WL.Config("cluster-L1000", L=1000, d=8, Nr=64, Nc=64, k=8, K=8, B=1, dtype=WL.F32),
    # the multi-kernel radix sort
    WL.Config("radix-M16384", L=1024, d=8, Nr=128, Nc=128, k=16, K=16, B=64, dtype=WL.F32),
]


@pytest.mark.parametrize("cfg", SCHED, ids=[c.name for c in SCHED])
def test_schedule_paths(cfg):
    """Every scheduler variant against the oracle on a seeded routing whose
    tokens share part of their experts."""
    idx, gate = WL.random_routing(cfg)
    ref = O.schedule(cfg, idx, gate.astype(np.float64))
    s = omni.schedule(omni.LayerDims.of(cfg), dev(idx), dev(gate))
    cnt = s["counts"].cpu().numpy()
    assert cnt[0] == ref["n_active"] and cnt[1] == ref["n_groups"] and cnt[2] == 0
    np.testing.assert_array_equal(s["task_token"].cpu().numpy(), ref["task_token"])
    np.testing.assert_array_equal(s["task_expert"].cpu().numpy(), ref["task_expert"])
    np.testing.assert_array_equal(s["task_gate"].cpu().numpy(), ref["task_gate"].astype(np.float32))
    np.testing.assert_array_equal(s["uniq"].cpu().numpy()[:cnt[0]], ref["uniq"])
    np.testing.assert_array_equal(s["group_off"].cpu().numpy()[:cnt[1] + 1], ref["group_off"])


def test_schedule_bad_index_sets_status():
    cfg = WL.TINY
    h = host_inputs(cfg)
    oi, og, _ = O.route(cfg, h)
    oi = oi.copy()
    oi[3, 2] = cfg.N + 5
    s = omni.schedule(omni.LayerDims.of(cfg), dev(oi), dev(og.astype(np.float32)))
    torch.cuda.synchronize()
    assert int(s["counts"][2].item()) & omni._lib.OMNI_DEV_BAD_INDEX


# --------------------------------------------------------------------------- execution


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_expert_forward_from_oracle_schedule(cfg):
    cs, h, d = sub_batch(cfg)
    oi, og, _ = O.route(cs, h)
    g32 = og.astype(np.float32)
    ref_s = O.schedule(cs, oi, g32.astype(np.float64))
    y_ref, rows = O.forward_expert(cs, h, ref_s)
    D = omni.LayerDims.of(cs)
    M = cs.L * cs.K
    counts = torch.tensor([ref_s["n_active"], ref_s["n_groups"], 0, 0], dtype=torch.int32,
                          device="cuda")
    sched = {"task_token": dev(ref_s["task_token"]), "task_expert": dev(ref_s["task_expert"]),
             "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
             "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]), "counts": counts}
    assert sched["task_token"].numel() == M
    y = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    err = rel_err(host_f64(y), y_ref)
    assert err <= tol_y(cs), err
    assert int(counts[2].item()) == 0


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_token_centric_from_oracle_routing(cfg):
    cs, h, d = sub_batch(cfg)
    oi, og, _ = O.route(cs, h)
    g32 = og.astype(np.float32)
    y_ref, _ = O.forward_token(cs, h, oi, g32.astype(np.float64))
    y = omni.token_centric_forward(omni.LayerDims.of(cs), d["x"], d["W"], d["V"], dev(oi),
                                   dev(g32))
    err = rel_err(host_f64(y), y_ref)
    assert err <= tol_y(cs), err


@pytest.mark.parametrize("cfg", ALL, ids=IDS)
def test_moe_forward_end_to_end(cfg):
    """The fused call on a sub-batch: routing ids as in test_route_end_to_end and
    y of every token whose ids match the oracle's."""
    cs, h, d = sub_batch(cfg)
    D = omni.LayerDims.of(cs)
    idx = torch.empty((cs.L, cs.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cs.L, cs.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         counts=counts, idx=idx, gate=gate)
    res = O.moe_forward(cs, h)
    _, _, bs, nxt = O.select_bruteforce(cs, *O.axis_logprobs(cs, h))
    gi = idx.cpu().numpy()
    lr, lc = O.axis_logprobs(cs, h)
    check_selection(cs, gi, gate.cpu().numpy(), None, res["idx"], res["gate"], res["score"], nxt,
                    lr, lc)
    same = np.all(np.sort(gi, 1) == np.sort(res["idx"], 1), axis=1)
    yg = host_f64(y)
    assert rel_err(yg[same], res["y"][same]) <= tol_y(cs)
    c = counts.cpu().numpy()
    assert c[2] == 0
    if same.all():
        assert c[0] == res["sched"]["n_active"] and c[1] == res["sched"]["n_groups"]


# ------------------------------------------------------------- full size (bench configuration)


@pytest.mark.parametrize("cfg", [WL.SKEWED, WL.PREFILL, WL.DECODE], ids=lambda c: c.name)
def test_full_size_fused_and_staged(cfg):
    """The whole batch as the benchmark runs it: the fused call against the staged
    calls, sampled rows against the oracle, and the schedule's defining
    properties checked on its own input at full size."""
    h = host_inputs(cfg)
    d = dev_inputs(cfg)
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         counts=counts, idx=idx, gate=gate)
    # staged
    i2, g2, _ = omni.route(D, d["x"], d["Wr"], d["Wc"], d["bias_r"], d["bias_c"])
    assert torch.equal(i2, idx) and torch.equal(g2, gate)
    s = omni.schedule(D, i2, g2)
    y2 = omni.expert_forward(D, d["x"], d["W"], d["V"], s)
    assert rel_err(host_f64(y2), host_f64(y)) <= 1e-2
    # schedule properties at full size, from its input: sorted by (group, token, expert)
    gi = i2.cpu().numpy().astype(np.int64)
    U = np.unique(gi)
    c = s["counts"].cpu().numpy()
    assert c[0] == len(U) and c[1] == (len(U) + cfg.B - 1) // cfg.B and c[2] == 0
    np.testing.assert_array_equal(s["uniq"].cpu().numpy()[:c[0]], U)
    t = np.repeat(np.arange(cfg.L), cfg.K)
    e = gi.reshape(-1)
    grp = np.searchsorted(U, e) // cfg.B
    order = np.lexsort((e, t, grp))
    np.testing.assert_array_equal(s["task_token"].cpu().numpy(), t[order])
    np.testing.assert_array_equal(s["task_expert"].cpu().numpy(), e[order])
    go = np.searchsorted(grp[order], np.arange(c[1] + 1))
    go[-1] = len(e)
    np.testing.assert_array_equal(s["group_off"].cpu().numpy()[:c[1] + 1], go)
    # sampled rows against the oracle
    tok = WL.sample_tokens(cfg, 128)
    cs = cfg.with_(L=len(tok))
    hs = dict(h, x=np.ascontiguousarray(h["x"][tok]))
    res = O.moe_forward(cs, hs)
    lr, lc = O.axis_logprobs(cs, hs)
    _, _, _, nxt = O.select_bruteforce(cs, lr, lc)
    gsub = gi[tok]
    check_selection(cs, gsub, gate.cpu().numpy()[tok], None, res["idx"], res["gate"],
                    res["score"], nxt, lr, lc)
    same = np.all(np.sort(gsub, 1) == np.sort(res["idx"], 1), axis=1)
    assert same.mean() > 0.5
    assert rel_err(host_f64(y)[tok][same], res["y"][same]) <= tol_y(cfg)


# --------------------------------------------------------------------------- edge cases

EDGE = [
    WL.Config("ragged-bf16", L=130, d=72, Nr=48, Nc=80, k=7, K=5, B=4, dtype=WL.BF16, seed=11),
    WL.Config("ragged-f32", L=37, d=40, Nr=12, Nc=20, k=9, K=9, B=2, dtype=WL.F32, seed=12),
    WL.Config("single-token", L=1, d=64, Nr=16, Nc=16, k=4, K=4, B=3, dtype=WL.BF16, seed=13),
    WL.Config("k1", L=200, d=128, Nr=32, Nc=64, k=1, K=1, B=5, dtype=WL.BF16, seed=14),
    WL.Config("max-topk", L=64, d=64, Nr=4096, Nc=256, k=256, K=256, B=64, dtype=WL.BF16, seed=15),
    WL.Config("wide-k", L=96, d=256, Nr=256, Nc=256, k=128, K=100, B=128, dtype=WL.BF16, seed=16),
]


@pytest.mark.parametrize("cfg", EDGE, ids=[c.name for c in EDGE])
def test_edge_shapes(cfg):
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], counts=counts, idx=idx,
                         gate=gate)
    res = O.moe_forward(cfg, h)
    lr, lc = O.axis_logprobs(cfg, h)
    _, _, _, nxt = O.select_bruteforce(cfg, lr, lc)
    gi = idx.cpu().numpy()
    check_selection(cfg, gi, gate.cpu().numpy(), None, res["idx"], res["gate"], res["score"], nxt,
                    lr, lc)
    same = np.all(np.sort(gi, 1) == np.sort(res["idx"], 1), axis=1)
    assert rel_err(host_f64(y)[same], res["y"][same]) <= tol_y(cfg)
    yt = omni.token_centric_forward(D, d["x"], d["W"], d["V"], idx, gate)
    assert rel_err(host_f64(yt), host_f64(y)) <= tol_y(cfg)


@pytest.mark.parametrize("L", [8, 300], ids=["one-cta-per-token", "two-warps-per-token"])
def test_equal_logits_pick_smallest_ids(L):
    """x = 0: every joint score ties; the K smallest ids of the k x k grid win
    (small batches take the 8-warp selection, larger ones the 2-warp one)."""
    cfg = WL.Config("ties", L=L, d=64, Nr=16, Nc=24, k=6, K=6, B=4, dtype=WL.BF16, seed=3)
    h = WL.make_inputs(cfg)
    h["x"] = np.zeros_like(h["x"])
    d = {k: dev(v) for k, v in h.items()}
    idx, gate, _ = omni.route(omni.LayerDims.of(cfg), d["x"], d["Wr"], d["Wc"])
    want = sorted(i * cfg.Nc + j for i in range(cfg.k) for j in range(cfg.k))[:cfg.K]
    assert np.all(idx.cpu().numpy() == np.array(want)[None, :])
    np.testing.assert_allclose(gate.cpu().numpy(), 1.0 / cfg.K, rtol=1e-6)


def test_empty_batch():
    cfg = WL.TINY.with_(L=0)
    D = omni.LayerDims.of(cfg)
    x = torch.empty((0, cfg.d), device="cuda")
    W = torch.zeros((cfg.N, cfg.d), device="cuda")
    y = omni.moe_forward(D, x, torch.zeros((cfg.Nr, cfg.d), device="cuda"),
                         torch.zeros((cfg.Nc, cfg.d), device="cuda"), W, W,
                         y=torch.empty((0, cfg.d), device="cuda"))
    assert y.shape == (0, cfg.d)


SWEEP = [
    WL.Config("sweeps-bf16", L=8192, d=2048, Nr=64, Nc=64, k=8, K=8, B=32, dtype=WL.BF16, seed=31),
    WL.Config("sweeps-f32", L=12288, d=1024, Nr=48, Nc=40, k=6, K=5, B=16, dtype=WL.F32, seed=32),
    # one group of all 49152 tasks: its window is larger than one CTA sorts
    WL.Config("sweeps-one-group", L=12288, d=1024, Nr=8, Nc=8, k=4, K=4, B=64, dtype=WL.BF16,
              seed=33),
]


@pytest.mark.parametrize("cfg", SWEEP, ids=[c.name for c in SWEEP])
def test_expert_sweeps_path(cfg):
    """Batches whose fp32 accumulator exceeds ~40 MiB run as an activation pass
    plus accumulation sweeps over column slices: same y as the oracle."""
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
    D = omni.LayerDims.of(cfg)
    assert cfg.L * cfg.d * 4 > (40 << 20)
    y = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)
    assert int(counts[2].item()) == 0


@pytest.mark.parametrize("flags", [omni.OMNI_FLAG_STAGED_SMALL, 0], ids=["windows", "default"])
@pytest.mark.parametrize("cfg", SWEEP, ids=[c.name for c in SWEEP])
def test_fused_sweeps_path(cfg, flags):
    """The fused forward of a sweep-sized batch goes from the routing straight
    to the window order of the sweeps (these batches' rows also fit in L2, so
    by default they take the routing-order tail; OMNI_FLAG_STAGED_SMALL keeps
    them on the window path): same y as the oracle's expert-centric execution
    of the routing it chose, same |U| and group count."""
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg, flags=flags)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         counts=counts, idx=idx, gate=gate)
    gi = idx.cpu().numpy()
    ref_s = O.schedule(cfg, gi, gate.cpu().numpy().astype(np.float64))
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    c = counts.cpu().numpy()
    assert c[0] == ref_s["n_active"] and c[1] == ref_s["n_groups"] and c[2] == 0
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)


def test_expert_sweeps_bad_group_count():
    """A group count on the device above its bound: the executor flags it
    (OMNI_DEV_BAD_INDEX) and still executes every task once, in schedule order."""
    cfg = SWEEP[0]
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    oi, og, _ = O.route(cfg, h)
    ref_s = O.schedule(cfg, oi, og.astype(np.float32).astype(np.float64))
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    D = omni.LayerDims.of(cfg)
    gmax = (min(cfg.N, cfg.L * cfg.K) + cfg.B - 1) // cfg.B
    counts = torch.tensor([ref_s["n_active"], gmax + 7, 0, 0], dtype=torch.int32, device="cuda")
    sched = {"task_token": dev(ref_s["task_token"]), "task_expert": dev(ref_s["task_expert"]),
             "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
             "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]), "counts": counts}
    y = omni.expert_forward(D, d["x"], d["W"], d["V"], sched)
    assert int(counts[2].item()) & omni._lib.OMNI_DEV_BAD_INDEX
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)


@pytest.mark.parametrize("cfg", [
    SWEEP[0],  # the window path of the fused forward
    # one CTA per token selects and clears the expert accumulator
    WL.Config("reuse-small", L=64, d=256, Nr=64, Nc=64, k=8, K=8, B=16, dtype=WL.BF16, seed=41),
], ids=lambda c: c.name)
def test_fused_workspace_reuse(cfg):
    """One workspace, filled with 0xFF before first use, serves two fused
    forwards of different batches: each equals a forward on a fresh workspace
    (nothing carries over from the workspace's earlier contents)."""
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    ws = omni.Workspace()
    ws.get(omni.workspace_size(D, omni._lib.OMNI_WS_FUSED), torch.device("cuda")).fill_(255)
    x2 = torch.roll(d["x"], shifts=7, dims=0).contiguous()
    ys = [omni.moe_forward(D, x, d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"], ws=ws)
          for x in (d["x"], x2)]
    for x, y in zip((d["x"], x2), ys):
        y_fresh = omni.moe_forward(D, x, d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"])
        assert rel_err(host_f64(y), host_f64(y_fresh)) <= tol_y(cfg)


def test_expert_sweeps_back_to_back():
    """Two grouped executions in a row on one workspace and stream, the second
    on other gates: the second's first clear of the accumulator slice must wait
    for the first call's last read of it."""
    cfg = SWEEP[0]
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    oi, og, _ = O.route(cfg, h)
    D = omni.LayerDims.of(cfg)
    ws = omni.Workspace()
    scheds, refs = [], []
    for scale in (1.0, -0.5):
        g32 = (og * scale).astype(np.float32)
        ref_s = O.schedule(cfg, oi, g32.astype(np.float64))
        refs.append(O.forward_expert(cfg, h, ref_s)[0])
        counts = torch.tensor([ref_s["n_active"], ref_s["n_groups"], 0, 0], dtype=torch.int32,
                              device="cuda")
        scheds.append({"task_token": dev(ref_s["task_token"]),
                       "task_expert": dev(ref_s["task_expert"]),
                       "task_gate": dev(ref_s["task_gate"].astype(np.float32)),
                       "uniq": dev(ref_s["uniq"]), "group_off": dev(ref_s["group_off"]),
                       "counts": counts})
    torch.cuda.synchronize()
    ys = [omni.expert_forward(D, d["x"], d["W"], d["V"], sc, ws=ws) for sc in scheds]
    torch.cuda.synchronize()
    for y, y_ref in zip(ys, refs):
        assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)


# --------------------- batches whose rows fit in L2: the two-kernel tail of the fused forward

SMALL_TAIL = [
    WL.Config("one-bf16-d256-L1", L=1, d=256, Nr=16, Nc=16, k=4, K=4, B=200, dtype=WL.BF16,
              seed=51),
    WL.Config("one-bf16-d512", L=37, d=512, Nr=40, Nc=30, k=16, K=16, B=7, dtype=WL.BF16, seed=52),
    WL.Config("one-bf16-d1024-skew", L=100, d=1024, Nr=64, Nc=64, k=8, K=8, B=64, dtype=WL.BF16,
              seed=53, zipf_s=1.1),
    WL.Config("one-f32-d128", L=50, d=128, Nr=32, Nc=32, k=6, K=6, B=16, dtype=WL.F32, seed=54),
    WL.Config("one-f32-d512", L=20, d=512, Nr=16, Nc=16, k=4, K=4, B=5, dtype=WL.F32, seed=55),
]


@pytest.mark.parametrize("cfg", SMALL_TAIL + [WL.DECODE], ids=lambda c: c.name)
def test_small_batch_tail(cfg):
    """The fused forward of a batch whose rows fit in L2 ends in two kernels
    (activations in routing order with a bitmap count of the active ids, then
    a per-token gather of the value rows): y against the oracle's
    expert-centric y of the same routing, |U| and the group count exactly,
    and y against the scheduling and execution kernels
    (OMNI_FLAG_STAGED_SMALL) on the same routing."""
    h = host_inputs(cfg) if cfg is WL.DECODE else WL.make_inputs(cfg)
    d = dev_inputs(cfg) if cfg is WL.DECODE else {k: dev(v) for k, v in h.items()}
    outs = {}
    for flags in (0, omni.OMNI_FLAG_STAGED_SMALL):
        D = omni.LayerDims.of(cfg, flags=flags)
        idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
        gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
        counts = omni.new_counts("cuda")
        y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"],
                             d["bias_c"], counts=counts, idx=idx, gate=gate)
        torch.cuda.synchronize()
        outs[flags] = (y.clone(), idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy())
    y1, i1, g1, c1 = outs[0]
    y2, i2, g2, c2 = outs[omni.OMNI_FLAG_STAGED_SMALL]
    assert np.array_equal(i1, i2) and np.array_equal(g1, g2)
    assert c1[2] == 0 and c2[2] == 0
    assert c1[0] == c2[0] and c1[1] == c2[1]
    assert rel_err(host_f64(y1), host_f64(y2)) <= tol_y(cfg)
    # against the oracle: its schedule of the GPU's routing, and y of that routing
    ref_s = O.schedule(cfg, i1, g1.astype(np.float64))
    assert c1[0] == ref_s["n_active"] and c1[1] == ref_s["n_groups"]
    y_ref, _ = O.forward_expert(cfg, h, ref_s)
    assert rel_err(host_f64(y1), y_ref) <= tol_y(cfg)
