"""GPU parity of the backward of the routed branch (omni_moe_backward)
against the oracle's fp64 backward, on the routing the GPU forward chose.

Bars (max|d - d_ref| / max|d_ref| per output):
- dW, dV: 1e-4 -- fp32 arithmetic on bf16-exact inputs, a few terms per row;
- dbias: 1e-3 -- fp32 sums of fp32 dS over the tokens, in atomic order;
- dx, dWr, dWc: 2e-2 -- the router's part goes through tensor-core products
  of bf16 operands (dZ rounded to bf16), fp32 accumulation.
The parameter gradients are added to what the caller passes: rows of experts
no token chose keep their values bit for bit.
"""
import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from helpers import dev, rel_err

pytestmark = pytest.mark.gpu

CONFIGS = [
    WL.Config("bwd-bf16-small", L=64, d=256, Nr=16, Nc=16, k=8, K=8, B=16, dtype=WL.BF16,
              seed=91),
    WL.Config("bwd-bf16-mid", L=1024, d=512, Nr=64, Nc=64, k=16, K=16, B=64, dtype=WL.BF16,
              seed=92),
    WL.Config("bwd-ragged", L=130, d=72, Nr=48, Nc=80, k=7, K=5, B=4, dtype=WL.BF16, seed=93),
    WL.Config("bwd-decode-shape", L=64, d=2048, Nr=128, Nc=128, k=64, K=64, B=128,
              dtype=WL.BF16, seed=94),
    WL.Config("bwd-skewed", L=512, d=256, Nr=32, Nc=32, k=8, K=8, B=32, dtype=WL.BF16, seed=95,
              zipf_s=1.1),
    # edges: one expert per token (the gate is 1, the router gets nothing);
    # the largest top-K (256 ids per token to search for each task's slot);
    # a single token
    WL.Config("bwd-k1", L=200, d=128, Nr=32, Nc=64, k=1, K=1, B=5, dtype=WL.BF16, seed=96),
    WL.Config("bwd-max-topk", L=64, d=64, Nr=4096, Nc=256, k=256, K=256, B=64, dtype=WL.BF16,
              seed=97),
    WL.Config("bwd-one-token", L=1, d=256, Nr=16, Nc=16, k=4, K=4, B=3, dtype=WL.BF16, seed=98),
]
TOL = {"dW": 1e-4, "dV": 1e-4, "dbias_r": 1e-3, "dbias_c": 1e-3, "dx": 2e-2, "dWr": 2e-2,
       "dWc": 2e-2}


def _bf16_dy(cfg):
    rng = np.random.default_rng(cfg.seed + 5)
    dy = torch.from_numpy(rng.standard_normal((cfg.L, cfg.d)).astype(np.float32))
    return dy.to(torch.bfloat16)


def _run(cfg, init=None):
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                     idx=idx, gate=gate)
    dy = _bf16_dy(cfg)
    grads = None if init is None else {k: v.clone() for k, v in init.items()}
    counts = omni.new_counts("cuda")
    g = omni.moe_backward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], idx, gate,
                          dy.cuda(), grads=grads, counts=counts)
    torch.cuda.synchronize()
    gi, gg = idx.cpu().numpy(), gate.cpu().numpy().astype(np.float64)
    ref = O.backward(cfg, h, gi, gg, dy.float().numpy().astype(np.float64))
    return h, g, ref, gi, counts.cpu().numpy()


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_backward_matches_the_oracle(cfg):
    _, g, ref, gi, c = _run(cfg)
    assert c[2] == 0
    assert c[0] == len(np.unique(gi))
    for key, tol in TOL.items():
        got = g[key].cpu().numpy().astype(np.float64)
        if not np.abs(ref[key]).max() > 0:  # K = 1: the router gets nothing
            assert np.abs(got).max() <= 1e-6, key
            continue
        err = rel_err(got, ref[key])
        assert err <= tol, (key, err)
    idle = np.setdiff1d(np.arange(cfg.N), gi)
    assert not g["dW"].cpu().numpy()[idle].any() and not g["dV"].cpu().numpy()[idle].any()


def test_backward_adds_to_the_given_gradients():
    cfg = CONFIGS[1]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3)
    init = {name: torch.randn(shape, generator=gen, device="cuda")
            for name, shape in (("dW", (cfg.N, cfg.d)), ("dV", (cfg.N, cfg.d)),
                                ("dWr", (cfg.Nr, cfg.d)), ("dWc", (cfg.Nc, cfg.d)),
                                ("dbias_r", (cfg.Nr,)), ("dbias_c", (cfg.Nc,)))}
    init["dx"] = torch.full((cfg.L, cfg.d), 5.0, device="cuda")  # overwritten
    _, g, ref, gi, c = _run(cfg, init)
    idle = np.setdiff1d(np.arange(cfg.N), gi)
    for key in ("dW", "dV"):
        base = init[key].cpu().numpy()
        got = g[key].cpu().numpy()
        assert np.array_equal(got[idle], base[idle])  # untouched rows, bit for bit
        assert rel_err(got.astype(np.float64) - base, ref[key]) <= 1e-4
    for key in ("dWr", "dWc", "dbias_r", "dbias_c"):
        got = g[key].cpu().numpy().astype(np.float64) - init[key].cpu().numpy()
        assert rel_err(got, ref[key]) <= TOL[key], key
    assert rel_err(g["dx"].cpu().numpy().astype(np.float64), ref["dx"]) <= TOL["dx"]


def test_backward_without_bias_gradients():
    cfg = CONFIGS[0]
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], idx=idx, gate=gate)
    g = omni.moe_backward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], idx, gate,
                          _bf16_dy(cfg).cuda(), bias=False)
    torch.cuda.synchronize()
    assert "dbias_r" not in g and "dbias_c" not in g
    ref = O.backward(cfg, h, idx.cpu().numpy(), gate.cpu().numpy().astype(np.float64),
                     _bf16_dy(cfg).float().numpy().astype(np.float64))
    assert rel_err(g["dWr"].cpu().numpy().astype(np.float64), ref["dWr"]) <= TOL["dWr"]


def test_backward_overwrites_without_reading():
    """accumulate=False: the active rows of dW, dV and the whole router and
    bias gradients are overwritten (what was there before does not matter,
    even NaN); rows of experts no token chose keep their values."""
    cfg = CONFIGS[4]
    init = {name: torch.full(shape, float("nan"), device="cuda")
            for name, shape in (("dW", (cfg.N, cfg.d)), ("dV", (cfg.N, cfg.d)),
                                ("dWr", (cfg.Nr, cfg.d)), ("dWc", (cfg.Nc, cfg.d)),
                                ("dbias_r", (cfg.Nr,)), ("dbias_c", (cfg.Nc,)))}
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                     idx=idx, gate=gate)
    dy = _bf16_dy(cfg)
    g = omni.moe_backward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], idx, gate, dy.cuda(),
                          grads={k: v.clone() for k, v in init.items()}, accumulate=False)
    torch.cuda.synchronize()
    gi = idx.cpu().numpy()
    ref = O.backward(cfg, h, gi, gate.cpu().numpy().astype(np.float64),
                     dy.float().numpy().astype(np.float64))
    act = np.unique(gi)
    idle = np.setdiff1d(np.arange(cfg.N), act)
    for key in ("dW", "dV"):
        got = g[key].cpu().numpy()
        assert np.isnan(got[idle]).all()
        assert rel_err(got[act].astype(np.float64), ref[key][act]) <= TOL[key]
    for key in ("dWr", "dWc", "dbias_r", "dbias_c", "dx"):
        got = g[key].cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all() and rel_err(got, ref[key]) <= TOL[key], key
