"""GPU parity of the shared dense MLP branch (two tcgen05 GEMMs) and of the
whole layer routed(x) + MLP(x), against the fp64 oracle.

Bar: max|dy| / max|y| <= 2e-2 (bf16 storage, fp32 accumulation; the hidden
activations are stored in bf16 between the two GEMMs and the fused layer
rounds the routed part to bf16 before the MLP is added -- each a relative
error of about 2^-9, well inside the bar)."""
import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from helpers import check_selection, dev, host_f64, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2

MLP_CASES = [
    # (config, F): single token, ragged tiles on every axis, K not a multiple
    # of 64, 128- and 256-wide B tiles, several waves of tiles
    (WL.Config("mlp-one-token", L=1, d=64, Nr=8, Nc=8, k=2, K=2, B=2, dtype=WL.BF16, seed=61), 64),
    (WL.Config("mlp-ragged", L=130, d=200, Nr=8, Nc=8, k=2, K=2, B=2, dtype=WL.BF16, seed=62), 328),
    (WL.Config("mlp-mid", L=300, d=512, Nr=8, Nc=8, k=2, K=2, B=2, dtype=WL.BF16, seed=63), 1024),
    (WL.Config("mlp-waves", L=4096, d=1024, Nr=8, Nc=8, k=2, K=2, B=2, dtype=WL.BF16, seed=64),
     2048),
]


def _mlp_inputs(cfg, F):
    h = WL.make_inputs(cfg, experts=False)
    h.update(WL.make_mlp(cfg, F))
    return h


@pytest.mark.parametrize("cfg,F", MLP_CASES, ids=[c.name for c, _ in MLP_CASES])
def test_shared_mlp_against_oracle(cfg, F):
    h = _mlp_inputs(cfg, F)
    d = {k: dev(h[k]) for k in ("x", "W1", "W2")}
    D = omni.LayerDims.of(cfg)
    counts = omni.new_counts("cuda")
    y = omni.shared_mlp(D, d["x"], d["W1"], d["W2"], counts=counts)
    tok = WL.sample_tokens(cfg, 256)
    ref = O.shared_mlp(cfg, h, h["W1"], h["W2"], tokens=tok)
    assert rel_err(host_f64(y)[tok], ref) <= TOL
    assert int(counts[2].item()) == 0
    # accumulate: y0 + MLP(x), one rounding of the sum
    y0 = torch.randn((cfg.L, cfg.d), device="cuda").bfloat16()
    y1 = omni.shared_mlp(D, d["x"], d["W1"], d["W2"], y=y0.clone(), accumulate=True)
    ref1 = host_f64(y0)[tok] + ref
    assert rel_err(host_f64(y1)[tok], ref1) <= TOL


@pytest.mark.parametrize("cfg,F", [
    (WL.Config("layer-small", L=64, d=256, Nr=32, Nc=32, k=8, K=8, B=16, dtype=WL.BF16, seed=65),
     512),
    (WL.Config("layer-mid", L=1024, d=512, Nr=64, Nc=64, k=8, K=8, B=32, dtype=WL.BF16, seed=66),
     1024),
], ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_layer_with_shared_mlp(cfg, F):
    """routed(x) + MLP(x) in one call against the oracle's routed output plus
    its MLP, on the tokens whose routing matches the oracle's."""
    h = _mlp_inputs(cfg, F)
    h.update(WL.make_experts(cfg))
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx = torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda")
    counts = omni.new_counts("cuda")
    y = omni.moe_mlp_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["W1"], d["W2"],
                             counts=counts, idx=idx, gate=gate)
    res = O.moe_forward(cfg, h)
    lr, lc = O.axis_logprobs(cfg, h)
    _, _, _, nxt = O.select_bruteforce(cfg, lr, lc)
    gi = idx.cpu().numpy()
    check_selection(cfg, gi, gate.cpu().numpy(), None, res["idx"], res["gate"], res["score"], nxt,
                    lr, lc)
    same = np.all(np.sort(gi, 1) == np.sort(res["idx"], 1), axis=1)
    ref = res["y"] + O.shared_mlp(cfg, h, h["W1"], h["W2"])
    assert rel_err(host_f64(y)[same], ref[same]) <= TOL
    c = counts.cpu().numpy()
    assert c[2] == 0 and c[0] == res["sched"]["n_active"] or not same.all()
