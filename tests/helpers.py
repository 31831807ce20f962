"""Shared helpers of the GPU parity tests (data movement and comparisons only)."""
import numpy as np
import torch

import workloads as WL


def dev(a, device="cuda"):
    """numpy array (bf16 as uint16 bits, or float32/int32) -> torch CUDA tensor."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host_f64(t):
    """torch tensor (bf16/f32/int) -> numpy float64 (bf16 widened exactly)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    return t.numpy().astype(np.float64)


def rel_err(y, ref):
    """max |y - ref| / max |ref|  (the layer-output parity metric)."""
    scale = float(np.abs(ref).max())
    return float(np.abs(y - ref).max()) / (scale if scale > 0 else 1.0)


def tol_y(cfg):
    return 1e-4 if cfg.dtype == WL.F32 else 2e-2


def check_selection(cfg, gpu_idx, gpu_gate, gpu_score, ora_idx, ora_gate, ora_score, nxt, lr, lc,
                    rel=1e-4, order_tol=1e-5):
    """Routing parity per token.

    Tokens whose oracle K-th and (K+1)-th best joint scores (over all N) are not a
    near-tie (gap >= rel * |S_K|) must select exactly the oracle's set of experts;
    gates and scores are compared expert by expert.  The order of the K outputs is
    (score desc, id asc) in each side's own arithmetic, so it is unique only where
    the scores are separated: the GPU order must agree with the oracle's wherever
    the oracle's scores differ by more than order_tol.  Near-tie tokens must hold a
    valid top-K within the tie band.  Returns (exact tokens, near-tie tokens).

    The band compares the oracle's K-th score with the (K+1)-th over all N
    joint scores (nxt).  That is the right pair only when k >= K: then the
    k x k candidates hold the true top-K, and a near-tie at the per-axis k-th
    place shows up as one at the K-th joint place.  The library refuses K > k
    where it selects, so a K > k configuration is a mistake in the test."""
    assert cfg.K <= cfg.k, "selection parity is defined for K <= k only"
    near = np.abs(ora_score[:, -1] - nxt) < rel * np.abs(ora_score[:, -1])
    exact = ~near
    gs = np.sort(gpu_idx, axis=1)
    os_ = np.sort(ora_idx, axis=1)
    bad = np.nonzero(exact & np.any(gs != os_, axis=1))[0]
    assert len(bad) == 0, f"{len(bad)} tokens select different experts, e.g. {bad[:5]}"
    for r in np.nonzero(exact)[0]:
        pos = {int(e): q for q, e in enumerate(ora_idx[r])}
        perm = np.array([pos[int(e)] for e in gpu_idx[r]])
        s_o = ora_score[r][perm]  # oracle score of each GPU output, in GPU order
        # a clearly worse expert may not come before a clearly better one
        later_best = np.maximum.accumulate(s_o[::-1])[::-1][1:]
        assert np.all(later_best <= s_o[:-1] + order_tol), f"token {r}: output order disagrees"
        np.testing.assert_allclose(gpu_gate[r], ora_gate[r][perm], rtol=2e-4, atol=2e-6)
        if gpu_score is not None:
            np.testing.assert_allclose(gpu_score[r], ora_score[r][perm], rtol=0, atol=2e-4)
    # near-tie tokens: the GPU set is a valid top-K of the oracle scores within the band
    for r in np.nonzero(near)[0]:
        e = gpu_idx[r].astype(np.int64)
        assert len(np.unique(e)) == cfg.K and e.min() >= 0 and e.max() < cfg.N
        s = lr[r, e // cfg.Nc] + lc[r, e % cfg.Nc]
        band = rel * abs(ora_score[r, -1])
        assert np.all(s >= ora_score[r, -1] - 2 * band)
        must = ora_idx[r][ora_score[r] > ora_score[r, -1] + 2 * band]
        assert set(must.tolist()) <= set(e.tolist())
        np.testing.assert_allclose(gpu_gate[r].sum(), 1.0, atol=1e-5)
    return int(exact.sum()), int(near.sum())
