"""GPU tests of the library as a runtime component: the forward captured in a
CUDA graph and replayed on new inputs, independent forwards on concurrent
streams, and a bounded device wait that runs out.

Every output is checked against the fp64 oracle as in the parity tests: the
routing ids bit-exact outside near-ties, and y against the oracle's
expert-centric execution of the routing the GPU chose.
"""
import time

import numpy as np
import pytest
import torch

import atomic_expert_routing_b200 as omni
import oracle as O
import workloads as WL
from atomic_expert_routing_b200 import _lib
from helpers import check_selection, dev, host_f64, rel_err, tol_y

pytestmark = pytest.mark.gpu

# a batch on the small-batch path and one on the window path of the sweeps
WINDOWS = WL.Config("graph-windows", L=8192, d=2048, Nr=64, Nc=64, k=8, K=8, B=32,
                    dtype=WL.BF16, seed=51)
CASES = [WL.TINY, WINDOWS]


def _other_x(cfg, seed):
    """x of another seed, same shape and distribution (the weights stay)."""
    return WL.make_inputs(cfg.with_(seed=seed), experts=False)["x"]


def _outputs(cfg):
    return (torch.empty((cfg.L, cfg.K), dtype=torch.int32, device="cuda"),
            torch.empty((cfg.L, cfg.K), dtype=torch.float32, device="cuda"),
            omni.new_counts("cuda"))


def _check_forward(cfg, h, y, idx, gate, counts):
    gi = idx.cpu().numpy()
    gg = gate.cpu().numpy()
    lr, lc = O.axis_logprobs(cfg, h)
    oi, og, os_ = O.select(cfg, lr, lc)
    _, _, _, nxt = O.select_bruteforce(cfg, lr, lc)
    exact, _ = check_selection(cfg, gi, gg, None, oi, og, os_, nxt, lr, lc)
    assert exact > 0.7 * cfg.L
    ref = O.schedule(cfg, gi, gg.astype(np.float64))
    y_ref, _ = O.forward_expert(cfg, h, ref)
    c = counts.cpu().numpy()
    assert c[0] == ref["n_active"] and c[1] == ref["n_groups"] and c[2] == 0
    assert rel_err(host_f64(y), y_ref) <= tol_y(cfg)


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_graph_replay_on_new_inputs(cfg):
    """One capture of the forward, replayed on two batches copied into its input
    buffer: each replay recomputes routing, schedule and y from the new x (y,
    ids and counters are cleared to garbage before each replay)."""
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx, gate, counts = _outputs(cfg)
    y = torch.empty((cfg.L, cfg.d), dtype=D.torch_dtype, device="cuda")
    x_in = d["x"].clone()
    ws = omni.Workspace()
    stream = torch.cuda.Stream()

    def fwd():
        omni.moe_forward(D, x_in, d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         y=y, counts=counts, idx=idx, gate=gate, ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        fwd()  # sizes the workspace outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fwd()
    for seed in (cfg.seed + 100, cfg.seed + 200):
        xs = _other_x(cfg, seed)
        x_in.copy_(dev(xs))
        y.fill_(float("nan"))
        idx.fill_(-1)
        counts.fill_(-7)
        counts[2] = 0  # the status word is sticky (OR): the caller clears it
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        _check_forward(cfg, dict(h, x=xs), y, idx, gate, counts)
    del g


def test_concurrent_streams():
    """Independent forwards on three streams, each with its own workspace,
    outputs and counters, launched back to back without synchronisation: the
    library keeps no state between calls, so each matches the oracle."""
    cfgs = [WINDOWS, WL.TINY, WL.BF16_16K.with_(L=2048)]
    runs = []
    for cfg in cfgs:
        h = WL.make_inputs(cfg)
        d = {k: dev(v) for k, v in h.items()}
        D = omni.LayerDims.of(cfg)
        idx, gate, counts = _outputs(cfg)
        y = torch.empty((cfg.L, cfg.d), dtype=D.torch_dtype, device="cuda")
        ws = omni.Workspace()
        ws.get(omni.workspace_size(D, _lib.OMNI_WS_FUSED), d["x"].device)
        runs.append((cfg, h, d, D, idx, gate, counts, y, ws, torch.cuda.Stream()))
    torch.cuda.synchronize()
    for cfg, h, d, D, idx, gate, counts, y, ws, s in runs:
        omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         y=y, counts=counts, idx=idx, gate=gate, ws=ws, stream=s)
    torch.cuda.synchronize()
    for cfg, h, d, D, idx, gate, counts, y, ws, s in runs:
        _check_forward(cfg, h, y, idx, gate, counts)


def test_bounded_wait_gives_up_and_reports():
    """A device wait that nothing completes gives up after its limit, sets
    OMNI_DEV_TIMEOUT in counts[2] and returns; the context stays usable, and
    a forward right after it on the same stream is correct and clean."""
    counts = omni.new_counts("cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    omni.wait_selftest(counts)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert counts.cpu().tolist() == [0, 0, _lib.OMNI_DEV_TIMEOUT, 0]
    assert 0.01 < waited < 60.0
    cfg = WL.TINY
    h = WL.make_inputs(cfg)
    d = {k: dev(v) for k, v in h.items()}
    D = omni.LayerDims.of(cfg)
    idx, gate, counts2 = _outputs(cfg)
    y = omni.moe_forward(D, d["x"], d["Wr"], d["Wc"], d["W"], d["V"], d["bias_r"], d["bias_c"],
                         counts=counts2, idx=idx, gate=gate)
    torch.cuda.synchronize()
    _check_forward(cfg, h, y, idx, gate, counts2)
