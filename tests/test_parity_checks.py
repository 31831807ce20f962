"""The comparisons the GPU parity tests rely on, checked on the CPU: fed the
oracle's own routing they pass, and fed a routing or an output with a planted
mistake they fail.  A checker that passed everything (every token flagged as
a near-tie, a tolerance that compares nothing) would make the GPU tests
vacuous."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from helpers import check_selection, dev, host_f64, rel_err, tol_y

CFG = WL.BF16_16K.with_(L=256)


@pytest.fixture(scope="module")
def routed():
    h = WL.make_inputs(CFG, experts=False)
    lr, lc = O.axis_logprobs(CFG, h)
    idx, gate, score = O.select(CFG, lr, lc)
    _, _, _, nxt = O.select_bruteforce(CFG, lr, lc)
    return idx, gate, score, nxt, lr, lc


def _check(routed, gi=None, gg=None, gs=None):
    idx, gate, score, nxt, lr, lc = routed
    gi = idx.copy() if gi is None else gi
    gg = gate.astype(np.float32) if gg is None else gg
    gs = score.astype(np.float32) if gs is None else gs
    return check_selection(CFG, gi, gg, gs, idx, gate, score, nxt, lr, lc)


def _separated_token(routed):
    """A token that is no near-tie and whose K scores are all distinct by a
    clear margin."""
    idx, gate, score, nxt, lr, lc = routed
    far = np.abs(score[:, -1] - nxt) > 1e-3 * np.abs(score[:, -1])
    ok = np.nonzero(far & (np.min(-np.diff(score, axis=1), axis=1) > 1e-4))[0]
    assert len(ok) > 0
    return int(ok[0])


def test_the_oracle_routing_passes(routed):
    exact, near = _check(routed)
    assert exact + near == CFG.L
    assert exact > 0.95 * CFG.L  # near-ties are rare on random logits


def test_the_output_order_is_checked_outside_ties_only(routed):
    """Swapping a token's first two outputs is an order error when their
    oracle scores are apart, and accepted when they tie (order within the
    tie is not unique)."""
    idx, gate, score, nxt, lr, lc = routed
    t = _separated_token(routed)
    gi, gg, gs = idx.copy(), gate.astype(np.float32).copy(), score.astype(np.float32).copy()
    for a in (gi, gg, gs):
        a[t, [0, 1]] = a[t, [1, 0]]
    with pytest.raises(AssertionError, match="order"):
        _check(routed, gi, gg, gs)
    tied = score.copy()
    tied[t, 1] = tied[t, 0]
    gs_t = tied.astype(np.float32).copy()
    gs_t[t, [0, 1]] = gs_t[t, [1, 0]]
    gate_t = gate.copy()
    gate_t[t, 1] = gate_t[t, 0]
    gg_t = gate_t.astype(np.float32).copy()
    gg_t[t, [0, 1]] = gg_t[t, [1, 0]]
    check_selection(CFG, gi, gg_t, gs_t, idx, gate_t, tied, nxt, lr, lc)


def test_a_wrong_expert_fails(routed):
    idx = routed[0]
    t = _separated_token(routed)
    gi = idx.copy()
    gi[t, -1] = (int(gi[t, -1]) + 1) % CFG.N
    while gi[t, -1] in idx[t]:
        gi[t, -1] = (int(gi[t, -1]) + 1) % CFG.N
    with pytest.raises(AssertionError):
        _check(routed, gi=gi)


def test_a_wrong_gate_or_score_fails(routed):
    t = _separated_token(routed)
    gg = routed[1].astype(np.float32).copy()
    gg[t, 0] *= 1.001
    with pytest.raises(AssertionError):
        _check(routed, gg=gg)
    gs = routed[2].astype(np.float32).copy()
    gs[t, 0] += 1e-3
    with pytest.raises(AssertionError):
        _check(routed, gs=gs)


def test_the_near_tie_band_accepts_a_valid_alternative_only(routed):
    """A token made a near-tie (its (K+1)-th score moved next to its K-th) may
    swap its K-th expert for another of the band, not for an arbitrary one."""
    idx, gate, score, nxt, lr, lc = routed
    t = _separated_token(routed)
    # the true (K+1)-th expert of token t, by brute force over all N
    S = (lr[t][:, None] + lc[t][None, :]).ravel()
    order = np.lexsort((np.arange(CFG.N), -S))
    alt = int(order[CFG.K])
    lr2, lc2 = lr.copy(), lc.copy()
    i, j = divmod(alt, CFG.Nc)
    # raise the alternative's row score so its joint score ties the K-th within the band
    lr2[t, i] += (score[t, -1] - S[alt]) * (1 - 1e-9)
    nxt2 = nxt.copy()
    nxt2[t] = lr2[t, i] + lc2[t, j]
    gi = idx.copy()
    gi[t, -1] = alt
    exact, near = check_selection(CFG, gi, gate.astype(np.float32), None, idx, gate, score, nxt2,
                                  lr2, lc2)
    assert near >= 1
    bad = idx.copy()
    bad[t, -1] = int(order[-1])  # the worst expert of all is outside the band
    with pytest.raises(AssertionError):
        check_selection(CFG, bad, gate.astype(np.float32), None, idx, gate, score, nxt2, lr2, lc2)


def test_output_tolerances():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((64, 128))
    assert rel_err(ref, ref) == 0.0
    bf16 = WL.BF16_16K
    assert rel_err(ref + 0.5 * tol_y(bf16) * np.abs(ref).max(), ref) <= tol_y(bf16)
    assert rel_err(ref + 2.0 * tol_y(bf16) * np.abs(ref).max(), ref) > tol_y(bf16)
    off = ref.copy()
    off[17, 33] += 2 * tol_y(WL.TINY) * np.abs(ref).max()  # one element is enough
    assert rel_err(off, ref) > tol_y(WL.TINY)
    assert tol_y(WL.TINY) == 1e-4 and tol_y(bf16) == 2e-2


def test_bf16_round_trip_of_the_data_movers():
    """bf16 bits go to a tensor and back to float64 exactly (CPU tensors)."""
    bits = np.array([[0x3F80, 0xC000, 0x4049, 0x0001]], np.uint16)
    t = dev(bits, device="cpu")
    assert t.dtype == torch.bfloat16
    np.testing.assert_array_equal(host_f64(t), WL.bf16_bits_to_f32(bits).astype(np.float64))
    assert dev(None) is None


def test_selection_check_refuses_K_above_k(routed):
    """The near-tie band compares the K-th and (K+1)-th joint scores over all
    N, which is only the selection's own margin when k >= K."""
    idx, gate, score, nxt, lr, lc = routed
    bad = CFG.with_(K=CFG.k + 1)
    with pytest.raises(AssertionError, match="K <= k"):
        check_selection(bad, idx, gate.astype(np.float32), score.astype(np.float32), idx, gate,
                        score, nxt, lr, lc)
