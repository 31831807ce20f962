"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a different
algorithm (brute force over all N joint scores), a closed form derived by
hand, a special case that reduces to a library routine (numpy/scipy), or an
invariant of the method.  The cases are chosen so that a plausible mistake
(a dropped log-softmax, a transposed router matrix, a swapped (i, j) -> id
mapping, a wrong SiLU sign, a V row mix-up, an unsorted schedule) fails one.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import expit, logsumexp, softmax
from scipy.special import log_softmax as scipy_log_softmax

import oracle as O
import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(a, cfg):
    return WL.bf16_bits_to_f32(a).astype(np.float64) if cfg.dtype == WL.BF16 else \
        np.asarray(a, np.float64)


def _small(**kw):
    base = dict(name="pin", L=24, d=16, Nr=6, Nc=9, k=4, K=4, B=3, dtype=WL.F32, seed=7)
    base.update(kw)
    return WL.Config(**base)


# --------------------------------------------------------------------------- router


@pytest.mark.parametrize("name", ["tiny-fp32", "bf16-N16K", "bf16-skewed-N256K",
                                  "bf16-prefill-N1M", "bf16-decode-N1M"])
def test_kxk_path_equals_bruteforce(name, inputs_cache):
    """Top-K over the k x k candidates equals top-K over all N joint scores when
    k >= K (per-axis dominance), index for index and gate for gate."""
    cfg = WL.CONFIGS[name]
    inp = inputs_cache(cfg, experts=False)
    tok = WL.sample_tokens(cfg, 512 if cfg.N <= 16384 else 128)
    lr, lc = O.axis_logprobs(cfg, inp, tok)
    idx, gate, score = O.select(cfg, lr, lc)
    bi, bg, bs, nxt = O.select_bruteforce(cfg, lr, lc)
    np.testing.assert_array_equal(idx, bi)
    np.testing.assert_allclose(gate, bg, rtol=0, atol=1e-15)
    np.testing.assert_allclose(score, bs, rtol=0, atol=0)
    # the K-th score beats the (K+1)-th (strict order by (S desc, e asc))
    assert np.all(bs[:, -1] >= nxt)


def test_row_log_softmax_matches_scipy():
    """The oracle's row-wise log-softmax (applied to logits the caller brings)
    against scipy's, on rows of different scales, and against the log-softmax
    the oracle's own routing applies to its axis logits."""
    rng = np.random.default_rng(5)
    z = rng.standard_normal((7, 33)) * np.array([1e-3, 1, 3, 10, 50, 200, 700])[:, None]
    np.testing.assert_allclose(O.log_softmax(z), scipy_log_softmax(z, axis=1), rtol=1e-14,
                               atol=1e-12)
    cfg = _small(L=12)
    inp = WL.make_inputs(cfg, experts=False)
    zr, zc = O.axis_logits(cfg, inp)
    lr, lc = O.axis_logprobs(cfg, inp)
    np.testing.assert_array_equal(O.log_softmax(zr), lr)
    np.testing.assert_array_equal(O.log_softmax(zc), lc)


def test_bruteforce_matches_numpy_sort():
    """The brute force against numpy on all N joint scores S = lr[i] + lc[j]
    (e = i*Nc + j): its K ids are np.lexsort's first K by (S desc, e asc), its
    scores are theirs, and its near-tie reference is the (K+1)-th best score."""
    for cfg in (_small(L=16), _small(L=16, k=4, K=7), WL.TINY.with_(L=16)):
        inp = WL.make_inputs(cfg, experts=False)
        lr, lc = O.axis_logprobs(cfg, inp)
        idx, _, score, nxt = O.select_bruteforce(cfg, lr, lc)
        S = (lr[:, :, None] + lc[:, None, :]).reshape(cfg.L, cfg.N)
        ids = np.arange(cfg.N)
        for t in range(cfg.L):
            order = np.lexsort((ids, -S[t]))
            np.testing.assert_array_equal(idx[t], order[:cfg.K])
            np.testing.assert_array_equal(score[t], S[t, order[:cfg.K]])
            assert nxt[t] == S[t, order[cfg.K]]


@pytest.mark.parametrize("name", ["tiny-fp32", "bf16-N16K", "bf16-skewed-N256K",
                                  "bf16-decode-N1M"])
def test_gates_sum_to_one_and_are_ordered(name, inputs_cache):
    cfg = WL.CONFIGS[name]
    inp = inputs_cache(cfg, experts=False)
    tok = WL.sample_tokens(cfg, 256)
    idx, gate, score = O.route(cfg, inp, tok)
    np.testing.assert_allclose(gate.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(gate > 0)
    # outputs ordered by (score desc, id asc); gates follow the scores
    assert np.all(np.diff(score, axis=1) <= 0)
    tie = np.diff(score, axis=1) == 0
    assert np.all(np.diff(idx, axis=1)[tie] > 0)
    assert np.all(np.diff(gate, axis=1) <= 1e-15)
    # gate ratio equals exp of score difference (softmax of the joint scores)
    np.testing.assert_allclose(gate / gate[:, :1], np.exp(score - score[:, :1]), rtol=1e-12)


def test_K1_is_argmax_of_each_axis():
    """k = K = 1: the expert is (argmax row logit, argmax column logit), gate 1.
    Reference: numpy matmul + argmax on the raw logits; Nr != Nc so a swapped
    (i, j) -> id mapping or a transposed router matrix fails."""
    cfg = _small(k=1, K=1, L=64)
    inp = WL.make_inputs(cfg, experts=False)
    x, Wr, Wc = (_f64(inp[n], cfg) for n in ("x", "Wr", "Wc"))
    idx, gate, _ = O.route(cfg, inp)
    i_ref = np.argmax(x @ Wr.T, axis=1)
    j_ref = np.argmax(x @ Wc.T, axis=1)
    np.testing.assert_array_equal(idx[:, 0], i_ref * cfg.Nc + j_ref)
    np.testing.assert_array_equal(gate, 1.0)


def test_select_all_is_the_product_distribution():
    """Brute force with K = N selects every expert; its scores are log(pr_i pc_j)
    and its gates pr_i * pc_j, with pr, pc the per-axis softmax (scipy)."""
    cfg = _small(L=8)
    inp = WL.make_inputs(cfg, experts=False)
    x, Wr, Wc = (_f64(inp[n], cfg) for n in ("x", "Wr", "Wc"))
    lr, lc = O.axis_logprobs(cfg, inp)
    full = cfg.with_(K=cfg.N, k=min(cfg.Nr, cfg.Nc))
    idx, gate, score, nxt = O.select_bruteforce(full, lr, lc)
    pr = softmax(x @ Wr.T, axis=1)
    pc = softmax(x @ Wc.T, axis=1)
    prod = (pr[:, :, None] * pc[:, None, :]).reshape(cfg.L, cfg.N)
    for t in range(cfg.L):
        np.testing.assert_allclose(gate[t], prod[t, idx[t]], rtol=1e-12)
        np.testing.assert_allclose(score[t], np.log(prod[t, idx[t]]), rtol=0, atol=1e-12)
        assert sorted(idx[t].tolist()) == list(range(cfg.N))
    assert np.all(np.isinf(nxt))
    np.testing.assert_allclose(logsumexp(score, axis=1), 0.0, atol=1e-12)


def test_hand_worked_example():
    """A 2 x 2 grid worked by hand (d = 2, fp32 storage).

    x = (1, 0).  Row keys give row logits (ln 3, 0): pr = (3/4, 1/4).
    Column keys give column logits (0, ln 2): pc = (1/3, 2/3).
    Joint probabilities (e = i*Nc + j): e0 = 1/4, e1 = 1/2, e2 = 1/12, e3 = 1/6.
    With k = K = 2: rows {0, 1}, columns {1, 0}; the best two are e1, e0,
    scores log(1/2), log(1/4), gates (1/2)/(3/4) = 2/3 and 1/3.
    Experts: W[1] = (a, 0), W[0] = (b, 0) with a = ln 3, b = -2, so
    h1 = SiLU(ln 3) = ln3 / (1 + 1/3) = (3/4) ln 3, h0 = -2 / (1 + e^2).
    V[1] = (1, 0), V[0] = (0, 1):  y = (2/3 * (3/4) ln 3, 1/3 * (-2/(1+e^2))).
    """
    ln3, ln2 = math.log(3.0), math.log(2.0)
    cfg = WL.Config("hand", L=1, d=2, Nr=2, Nc=2, k=2, K=2, B=2, dtype=WL.F32)
    f = lambda a: np.ascontiguousarray(a, np.float32)
    inp = {
        "x": f([[1.0, 0.0]]),
        "Wr": f([[ln3, 0.0], [0.0, 0.0]]),
        "Wc": f([[0.0, 0.0], [ln2, 0.0]]),
        "W": f([[-2.0, 0.0], [ln3, 0.0], [0.0, 0.0], [0.0, 0.0]]),
        "V": f([[0.0, 1.0], [1.0, 0.0], [0.0, 0.0], [0.0, 0.0]]),
        "bias_r": None, "bias_c": None,
    }
    # the fp32-stored values of ln 3 and ln 2 (what the oracle reads)
    l3, l2 = float(np.float32(ln3)), float(np.float32(ln2))
    pr = np.exp([l3, 0.0]) / (math.exp(l3) + 1.0)
    pc = np.exp([0.0, l2]) / (1.0 + math.exp(l2))
    idx, gate, score = O.route(cfg, inp)
    assert idx.tolist() == [[1, 0]]
    np.testing.assert_allclose(score[0], [math.log(pr[0] * pc[1]), math.log(pr[0] * pc[0])],
                               atol=1e-14)
    np.testing.assert_allclose(gate[0], [2 / 3, 1 / 3], atol=1e-7)   # fp32-stored ln's
    np.testing.assert_allclose(gate[0], [pc[1], pc[0]], atol=1e-14)  # exact for stored ln 2
    sched = O.schedule(cfg, idx, gate)
    y, rows = O.forward_expert(cfg, inp, sched)
    h1 = l3 / (1 + math.exp(-l3))
    h0 = -2.0 / (1 + math.exp(2.0))
    np.testing.assert_allclose(y[0], [gate[0, 0] * h1, gate[0, 1] * h0], atol=1e-15)
    np.testing.assert_allclose(y[0], [2 / 3 * 0.75 * ln3, 1 / 3 * (-2 / (1 + math.e ** 2))],
                               atol=1e-7)
    assert rows == (2, 2)


# bf16 bit patterns and their values, decoded by hand from the format (1 sign
# bit, 8 exponent bits with bias 127, 7 mantissa bits)
_BF16_HAND = [
    (0x3F80, 1.0),
    (0xC000, -2.0),
    (0x4049, 3.140625),                     # 2 * (1 + 73/128)
    (0x3F81, 1.0078125),                    # 1 + 2^-7
    (0xBE80, -0.25),                        # exponent 125
    (0x0001, 2.0 ** -133),                  # smallest subnormal: 2^-7 * 2^-126
    (0x7F7F, 2.0 ** 127 * 255 / 128),       # largest finite
    (0x8000, -0.0),
]


def test_bf16_widening_and_rounding_of_the_input_generator():
    """The shared input generator's bf16 helpers against hand-decoded values:
    exact widening, and round-to-nearest with ties to even."""
    bits = np.array([b for b, _ in _BF16_HAND], np.uint16)
    vals = WL.bf16_bits_to_f32(bits).astype(np.float64)
    for (b, want), got in zip(_BF16_HAND, vals):
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), hex(b)
    np.testing.assert_array_equal(WL.f32_to_bf16_bits(vals.astype(np.float32)), bits)
    f = np.array([1.0 + 2.0 ** -8,                # half-way, 0x3F80 is even
                  1.0 + 3 * 2.0 ** -8,            # half-way, 0x3F82 is even
                  1.0 + 2.0 ** -8 + 2.0 ** -20,   # just above half-way
                  -(1.0 + 2.0 ** -8 - 2.0 ** -20),  # just below half-way, negative
                  float(np.float32(math.pi))], np.float32)
    np.testing.assert_array_equal(WL.f32_to_bf16_bits(f),
                                  np.array([0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x4049], np.uint16))


def test_bf16_storage_is_read_exactly():
    """bf16-stored operands enter the oracle at their exact values: with x = 1
    (d = 1) each raw row logit is the hand-decoded value of one stored key."""
    cfg = WL.Config("bits", L=1, d=1, Nr=len(_BF16_HAND), Nc=2, k=1, K=1, B=1, dtype=WL.BF16)
    inp = {
        "x": np.array([[0x3F80]], np.uint16),
        "Wr": np.array([[b] for b, _ in _BF16_HAND], np.uint16),
        "Wc": np.array([[0x3F80], [0xC000]], np.uint16),
    }
    zr, zc = O.axis_logits(cfg, inp)
    np.testing.assert_array_equal(zr[0], [v for _, v in _BF16_HAND])
    np.testing.assert_array_equal(zc[0], [1.0, -2.0])


def test_bf16_router_logits_match_numpy():
    """Raw router logits of a bf16 workload against numpy's x @ Wr^T on the
    widened operands (Nr != Nc, so a transposed router matrix fails too)."""
    cfg = _small(dtype=WL.BF16, d=96, L=40)
    inp = WL.make_inputs(cfg, experts=False)
    x, Wr, Wc = (_f64(inp[n], cfg) for n in ("x", "Wr", "Wc"))
    zr, zc = O.axis_logits(cfg, inp)
    np.testing.assert_allclose(zr, x @ Wr.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(zc, x @ Wc.T, rtol=1e-13, atol=1e-13)


def test_equal_logits_break_ties_by_smaller_id():
    """x = 0 makes every logit equal: all joint scores tie, the K smallest ids
    of the k x k candidate grid win (rows 0.., columns 0..), gates are 1/K."""
    cfg = _small(k=3, K=5, L=4)
    inp = WL.make_inputs(cfg, experts=False)
    inp["x"] = np.zeros_like(inp["x"])
    idx, gate, score = O.route(cfg, inp)
    want = sorted(i * cfg.Nc + j for i in range(cfg.k) for j in range(cfg.k))[: cfg.K]
    for t in range(cfg.L):
        assert idx[t].tolist() == want
    np.testing.assert_allclose(gate, 1.0 / cfg.K, atol=1e-15)
    np.testing.assert_allclose(score, -math.log(cfg.Nr) - math.log(cfg.Nc), atol=1e-14)


def test_bias_shift_invariance_and_bias_sign():
    """A constant added to every row bias (or column bias) cancels in the
    per-axis log-softmax; a large bias on row a / column b forces expert
    a*Nc + b to the top with gate near 1."""
    cfg = _small(L=32)
    inp = WL.make_inputs(cfg, experts=False)
    z = dict(inp)
    z["bias_r"] = np.zeros(cfg.Nr, np.float32)
    z["bias_c"] = np.zeros(cfg.Nc, np.float32)
    i0, g0, s0 = O.route(cfg, z)
    z["bias_r"] = np.full(cfg.Nr, 3.25, np.float32)
    z["bias_c"] = np.full(cfg.Nc, -7.5, np.float32)
    i1, g1, s1 = O.route(cfg, z)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_allclose(g0, g1, atol=1e-13)
    np.testing.assert_allclose(s0, s1, atol=1e-12)
    z["bias_r"] = np.zeros(cfg.Nr, np.float32)
    z["bias_c"] = np.zeros(cfg.Nc, np.float32)
    z["bias_r"][4] = 60.0
    z["bias_c"][7] = 60.0
    i2, g2, s2 = O.route(cfg, z)
    assert np.all(i2[:, 0] == 4 * cfg.Nc + 7)
    assert np.all(g2[:, 0] > 1 - 1e-12)


def test_router_cost_ratio_golden():
    """(Nr + Nc) / N at N = 16K with a square grid is the printed 1.56%."""
    vals = {}
    with open(os.path.join(GOLDEN, "router_cost.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    cfg = WL.BF16_16K
    assert (cfg.N, cfg.Nr, cfg.Nc) == (vals["N"], vals["Nr"], vals["Nc"])
    ratio = 100.0 * (cfg.Nr + cfg.Nc) / cfg.N
    assert ratio == 1.5625
    assert round(ratio, 2) == vals["ratio_percent_printed"]
    assert cfg.Nr == math.isqrt(cfg.N)


# --------------------------------------------------------------------------- schedule


def _reference_order(idx, gate, tok, B):
    """The schedule's definition written with library primitives:
    np.unique (sorted unique ids), searchsorted (rank), np.lexsort."""
    K = idx.shape[1]
    t = np.repeat(tok, K)
    e = idx.reshape(-1).astype(np.int64)
    g = gate.reshape(-1)
    U = np.unique(e)
    grp = np.searchsorted(U, e) // B
    order = np.lexsort((e, t, grp))
    go = np.searchsorted(grp[order], np.arange((len(U) + B - 1) // B + 1), side="left")
    go[-1] = len(e)
    return t[order], e[order], g[order], U, go


@pytest.mark.parametrize("name,B", [("tiny-fp32", None), ("bf16-N16K", None),
                                    ("tiny-fp32", 1), ("tiny-fp32", 10 ** 6),
                                    ("bf16-skewed-N256K", None), ("bf16-decode-N1M", None)])
def test_schedule_matches_library_definition(name, B, inputs_cache):
    cfg = WL.CONFIGS[name]
    if B is not None:
        cfg = cfg.with_(B=B)
    inp = inputs_cache(cfg.with_(B=WL.CONFIGS[name].B), experts=False)
    tok = WL.sample_tokens(cfg, 1024)
    idx, gate, _ = O.route(cfg, inp, tok)
    s = O.schedule(cfg, idx, gate, tok)
    tt, te, tg, U, go = _reference_order(idx, gate, tok, cfg.B)
    np.testing.assert_array_equal(s["task_token"], tt)
    np.testing.assert_array_equal(s["task_expert"], te)
    np.testing.assert_array_equal(s["task_gate"], tg)
    np.testing.assert_array_equal(s["uniq"], U)
    np.testing.assert_array_equal(s["group_off"], go)
    assert s["n_active"] == len(U)
    assert s["n_groups"] == (len(U) + cfg.B - 1) // cfg.B
    # structural invariants
    assert np.all(np.diff(s["uniq"]) > 0)
    assert np.all(np.diff(s["group_off"]) > 0)  # no empty group
    for g in range(s["n_groups"]):
        seg = s["task_expert"][s["group_off"][g]:s["group_off"][g + 1]]
        assert len(np.unique(seg)) <= cfg.B
        assert set(np.unique(seg)) == set(s["uniq"][g * cfg.B:(g + 1) * cfg.B])
    if cfg.B == 1:
        assert s["n_groups"] == s["n_active"]
    if cfg.B >= s["n_active"]:
        assert s["n_groups"] == 1


# --------------------------------------------------------------------------- execution


@pytest.mark.parametrize("name", ["tiny-fp32", "bf16-N16K", "bf16-skewed-N256K"])
def test_expert_centric_equals_token_centric(name, inputs_cache):
    """Both execution orders compute the same layer output (the scheduling is a
    pure reordering); row counters equal the traffic model 2d*|E| vs 2d*L*K."""
    cfg = WL.CONFIGS[name]
    inp = inputs_cache(cfg, experts=True)
    tok = WL.sample_tokens(cfg, 512)
    idx, gate, _ = O.route(cfg, inp, tok)
    s = O.schedule(cfg, idx, gate, tok)
    ye, re = O.forward_expert(cfg, inp, s, tok)
    yt, rt = O.forward_token(cfg, inp, idx, gate, tok)
    scale = np.abs(yt).max()
    assert scale > 0
    assert np.abs(ye - yt).max() <= 1e-12 * scale
    M = len(tok) * cfg.K
    assert re == (s["n_active"], s["n_active"])
    assert rt == (M, M)
    d_tok = cfg.d * (rt[0] + rt[1])
    d_exp = cfg.d * (re[0] + re[1])
    assert d_tok == 2 * cfg.d * len(tok) * cfg.K
    assert d_exp == 2 * cfg.d * s["n_active"]
    assert d_exp <= d_tok


def _manual_schedule(cfg, idx, gate):
    tok = np.arange(idx.shape[0], dtype=np.int64)
    return O.schedule(cfg, idx, gate, tok)


def test_one_hot_value_rows_recover_gate_times_silu():
    """V[e] = one-hot at column (e mod d): y[t, c] = sum over t's experts with
    e mod d = c of gate * SiLU(x[t] . W[e]); h from numpy dot + scipy expit."""
    cfg = WL.Config("probe", L=16, d=32, Nr=8, Nc=8, k=4, K=5, B=4, dtype=WL.F32, seed=3)
    inp = WL.make_inputs(cfg)
    V = np.zeros((cfg.N, cfg.d), np.float32)
    V[np.arange(cfg.N), np.arange(cfg.N) % cfg.d] = 1.0
    inp = dict(inp, V=V)
    idx, gate, _ = O.route(cfg, inp)
    y, _ = O.forward_expert(cfg, inp, _manual_schedule(cfg, idx, gate))
    x, W = inp["x"].astype(np.float64), inp["W"].astype(np.float64)
    ref = np.zeros((cfg.L, cfg.d))
    for t in range(cfg.L):
        for q in range(cfg.K):
            e = idx[t, q]
            z = float(np.dot(x[t], W[e]))
            ref[t, e % cfg.d] += gate[t, q] * z * expit(z)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-14)


def test_execution_closed_forms():
    """Hand-made tasks: x[t] = s_t * e_0 and W[e] = a_e * e_0 give
    x . W[e] = s_t a_e exactly; SiLU(z) = z / (1 + e^-z) with its sign;
    x = 0 gives y = 0; scaling V scales y (linearity, sign of V)."""
    cfg = WL.Config("closed", L=3, d=8, Nr=2, Nc=3, k=2, K=2, B=2, dtype=WL.F32)
    x = np.zeros((3, 8), np.float32)
    x[:, 0] = [1.0, -1.5, 0.0]
    W = np.zeros((6, 8), np.float32)
    W[:, 0] = [2.0, -2.0, 0.5, 1.0, -0.25, 3.0]
    V = np.zeros((6, 8), np.float32)
    V[np.arange(6), [1, 2, 3, 4, 5, 6]] = [1.0, 2.0, -1.0, 0.5, 4.0, -3.0]
    inp = {"x": x, "W": W, "V": V}
    idx = np.array([[1, 5], [0, 4], [2, 3]], np.int32)
    gate = np.array([[0.75, 0.25], [0.5, 0.5], [0.9, 0.1]])
    sched = _manual_schedule(cfg, idx, gate)
    y, _ = O.forward_expert(cfg, inp, sched)
    silu = lambda z: z / (1.0 + math.exp(-z))
    ref = np.zeros((3, 8))
    ref[0, 2] = 0.75 * silu(1.0 * -2.0) * 2.0
    ref[0, 6] = 0.25 * silu(1.0 * 3.0) * -3.0
    ref[1, 1] = 0.5 * silu(-1.5 * 2.0) * 1.0
    ref[1, 5] = 0.5 * silu(-1.5 * -0.25) * 4.0
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-15)
    assert silu(-2.0) < 0 < silu(3.0)
    assert np.all(y[2] == 0.0)  # x = 0 -> SiLU(0) = 0
    y2, _ = O.forward_expert(cfg, dict(inp, V=-2 * V), sched)
    np.testing.assert_allclose(y2, -2 * y, rtol=0, atol=1e-15)
    yt, _ = O.forward_token(cfg, inp, idx, gate)
    np.testing.assert_allclose(yt, ref, rtol=0, atol=1e-15)


def test_thread_count_does_not_change_results():
    """The oracle's OpenMP loops split independent tokens (and ids): one thread
    and all threads give bit-identical routing and y."""
    cfg = WL.TINY
    h = WL.make_inputs(cfg)
    a = O.moe_forward(cfg, h)
    n = O.num_threads()
    try:
        O.set_num_threads(1)
        assert O.num_threads() == 1
        b = O.moe_forward(cfg, h)
    finally:
        O.set_num_threads(n)
    for k in ("idx", "gate", "score", "y"):
        np.testing.assert_array_equal(np.asarray(a[k]), np.asarray(b[k]))


# ------------------------------------------------------------ shared dense MLP branch

def _mlp_cfg(L, d, dtype=WL.F32):
    return WL.Config("mlp", L=L, d=d, Nr=2, Nc=2, k=1, K=1, B=1, dtype=dtype, seed=0)


def test_shared_mlp_hand_worked():
    """d = 2, F = 3, two tokens; the numbers are worked by hand.
    Token 0, x = (1, -2): x W1^T = (1, -2, -1), SiLU of those
    = (sigmoid(1), -2 sigmoid(-2), -sigmoid(-1)) = (0.7310585786, -0.2384058440,
    -0.2689414214); with W2 rows (1, -1, 2) and (0, 3, 0.5) the outputs are
    (0.4315815799, -0.8496882428).  Token 1, x = (0.5, 0): x W1^T = (0.5, 0,
    0.5), SiLU = (0.3112296656, 0, 0.3112296656), outputs (0.9336889968,
    0.1556148328)."""
    cfg = _mlp_cfg(2, 2)
    x = np.array([[1.0, -2.0], [0.5, 0.0]], np.float32)
    W1 = np.array([[1, 0], [0, 1], [1, 1]], np.float32)
    W2 = np.array([[1, -1, 2], [0, 3, 0.5]], np.float32)
    y = O.shared_mlp(cfg, {"x": x}, W1, W2)
    ref = np.array([[0.4315815799, -0.8496882428], [0.9336889968, 0.1556148328]])
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-9)


@pytest.mark.parametrize("dtype", [WL.F32, WL.BF16], ids=["f32", "bf16"])
def test_shared_mlp_identity_output_is_silu_of_the_projection(dtype):
    """With F = d and W2 = I the branch is SiLU(x W1^T), element by element:
    numpy's matmul and scipy's expit in fp64 on the exact stored values."""
    cfg = _mlp_cfg(7, 24, dtype)
    rng = np.random.default_rng(5)
    x32 = rng.standard_normal((7, 24)).astype(np.float32)
    W132 = (rng.standard_normal((24, 24)) / 5).astype(np.float32)
    if dtype == WL.BF16:
        x, W1 = WL.f32_to_bf16_bits(x32), WL.f32_to_bf16_bits(W132)
        W2 = WL.f32_to_bf16_bits(np.eye(24, dtype=np.float32))
        xf, W1f = WL.bf16_bits_to_f32(x), WL.bf16_bits_to_f32(W1)
    else:
        x, W1, W2, xf, W1f = x32, W132, np.eye(24, dtype=np.float32), x32, W132
    y = O.shared_mlp(cfg, {"x": x}, W1, W2)
    z = xf.astype(np.float64) @ W1f.astype(np.float64).T
    np.testing.assert_allclose(y, z * expit(z), rtol=1e-12, atol=1e-14)


def test_shared_mlp_linearity_rows_and_zero():
    """Linear in W2; every token depends on its own row of x only (a token
    subset gives those rows); x = 0 gives 0 (SiLU(0) = 0)."""
    cfg = _mlp_cfg(9, 16)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((9, 16)).astype(np.float32)
    x[4] = 0.0
    W1 = (rng.standard_normal((40, 16)) / 4).astype(np.float32)
    # dyadic weights: 2 W2a - 3 W2b is exact in fp32
    W2a = (rng.integers(-8, 9, (16, 40)) / 64).astype(np.float32)
    W2b = (rng.integers(-8, 9, (16, 40)) / 64).astype(np.float32)
    ya = O.shared_mlp(cfg, {"x": x}, W1, W2a)
    yb = O.shared_mlp(cfg, {"x": x}, W1, W2b)
    yab = O.shared_mlp(cfg, {"x": x}, W1, (2 * W2a - 3 * W2b).astype(np.float32))
    np.testing.assert_allclose(yab, 2 * ya - 3 * yb, rtol=1e-12, atol=1e-12)
    assert np.all(ya[4] == 0.0)
    tok = np.array([1, 4, 8], np.int64)
    np.testing.assert_array_equal(O.shared_mlp(cfg, {"x": x}, W1, W2a, tokens=tok), ya[tok])


# ------------------------------------------------------------ gated (SwiGLU) atomic expert

def test_gated_expert_hand_worked():
    """The closed-form tasks above with a gate matrix: U[e] = b_e * e_7 and
    x[t, 7] = (2, 1, 5), so x . U[e] = x7_t b_e and h = SiLU(s_t a_e) x7_t b_e.
    Worked by hand: token 0 -> expert 1 (a = -2, b = 0.5) and expert 5 (a = 3,
    b = -0.5); token 1 -> expert 0 (a = 2, b = 1) and expert 4 (a = -0.25,
    b = 4); token 2 has s = 0, so SiLU(0) = 0 and its row stays 0."""
    cfg = WL.Config("closed-glu", L=3, d=8, Nr=2, Nc=3, k=2, K=2, B=2, dtype=WL.F32)
    x = np.zeros((3, 8), np.float32)
    x[:, 0] = [1.0, -1.5, 0.0]
    x[:, 7] = [2.0, 1.0, 5.0]
    W = np.zeros((6, 8), np.float32)
    W[:, 0] = [2.0, -2.0, 0.5, 1.0, -0.25, 3.0]
    U = np.zeros((6, 8), np.float32)
    U[:, 7] = [1.0, 0.5, -1.0, 2.0, 4.0, -0.5]
    V = np.zeros((6, 8), np.float32)
    V[np.arange(6), [1, 2, 3, 4, 5, 6]] = [1.0, 2.0, -1.0, 0.5, 4.0, -3.0]
    inp = {"x": x, "W": W, "U": U, "V": V}
    idx = np.array([[1, 5], [0, 4], [2, 3]], np.int32)
    gate = np.array([[0.75, 0.25], [0.5, 0.5], [0.9, 0.1]])
    sched = _manual_schedule(cfg, idx, gate)
    y, _ = O.forward_expert(cfg, inp, sched)
    ref = np.zeros((3, 8))
    ref[0, 2] = -0.3576087661   # 0.75 * SiLU(-2) * (2 * 0.5) * 2
    ref[0, 6] = 2.1432917854    # 0.25 * SiLU(3) * (2 * -0.5) * -3
    ref[1, 1] = -0.0711388098   # 0.5 * SiLU(-3) * (1 * 1) * 1
    ref[1, 5] = 1.7779997999    # 0.5 * SiLU(0.375) * (1 * 4) * 4
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-9)
    yt, _ = O.forward_token(cfg, inp, idx, gate)
    np.testing.assert_allclose(yt, ref, rtol=0, atol=1e-9)


def test_gated_expert_with_a_unit_gate_is_the_plain_expert():
    """A constant feature x[:, 0] = 1 and U[e] = e_0 make x . U[e] = 1 for every
    task: the gated expert reduces to the plain one (both orders)."""
    cfg = WL.TINY.with_(L=40)
    h = WL.make_inputs(cfg)
    x = WL.bf16_bits_to_f32(h["x"]) if cfg.dtype == WL.BF16 else h["x"].copy()
    x[:, 0] = 1.0
    U = np.zeros((cfg.N, cfg.d), np.float32)
    U[:, 0] = 1.0
    inp = dict(h, x=x.astype(np.float32))
    idx, gate, _ = O.route(cfg, inp)
    sched = O.schedule(cfg, idx, gate)
    y_plain, _ = O.forward_expert(cfg, inp, sched)
    y_glu, _ = O.forward_expert(cfg, dict(inp, U=U), sched)
    np.testing.assert_allclose(y_glu, y_plain, rtol=1e-12, atol=1e-14)
    yt, _ = O.forward_token(cfg, dict(inp, U=U), idx, gate)
    np.testing.assert_allclose(yt, y_plain, rtol=1e-12, atol=1e-14)


def test_gated_expert_linear_in_U_and_orders_agree():
    cfg = WL.TINY.with_(L=48)
    h = WL.make_inputs(cfg)
    rng = np.random.default_rng(8)
    U = (rng.integers(-8, 9, (cfg.N, cfg.d)) / 64).astype(np.float32)  # dyadic: 3U exact
    idx, gate, _ = O.route(cfg, h)
    sched = O.schedule(cfg, idx, gate)
    y1, _ = O.forward_expert(cfg, dict(h, U=U), sched)
    y3, _ = O.forward_expert(cfg, dict(h, U=(3 * U).astype(np.float32)), sched)
    np.testing.assert_allclose(y3, 3 * y1, rtol=1e-12, atol=1e-13)
    yt, _ = O.forward_token(cfg, dict(h, U=U), idx, gate)
    np.testing.assert_allclose(yt, y1, rtol=1e-12, atol=1e-13)
    assert np.abs(y1).max() > 0


# ------------------------------------------------------------------ backward
#
# The gradients are pinned to the oracle's forward, not to a second copy of
# their formulas: for the loss l = sum(dy * y), the central difference of l
# along a direction v of one input, (l(p + e v) - l(p - e v)), must equal
# <grad, p+ - p-> up to terms of third order in e, where p+- are the stored
# (fp32) perturbed inputs.  The selected sets must not change between the
# two evaluations (the selection is piecewise constant); the test asserts it.

BWD_CFGS = [
    WL.Config("bwd-tiny", L=4, d=8, Nr=5, Nc=4, k=3, K=3, B=2, dtype=WL.F32, seed=3),
    WL.Config("bwd-small", L=12, d=24, Nr=9, Nc=7, k=4, K=4, B=3, dtype=WL.F32, seed=4),
]


def _loss(cfg, h, dy):
    res = O.moe_forward(cfg, h)
    return float(np.sum(dy * res["y"])), res["idx"]


def _bias_inputs(cfg):
    h = WL.make_inputs(cfg)
    rng = np.random.default_rng(cfg.seed)
    h["bias_r"] = (0.3 * rng.standard_normal(cfg.Nr)).astype(np.float32)
    h["bias_c"] = (0.3 * rng.standard_normal(cfg.Nc)).astype(np.float32)
    return h


@pytest.mark.parametrize("cfg", BWD_CFGS, ids=lambda c: c.name)
@pytest.mark.parametrize("name,grad", [("x", "dx"), ("W", "dW"), ("V", "dV"), ("Wr", "dWr"),
                                       ("Wc", "dWc"), ("bias_r", "dbias_r"),
                                       ("bias_c", "dbias_c")])
def test_backward_matches_central_differences_of_the_forward(cfg, name, grad):
    h = _bias_inputs(cfg)
    rng = np.random.default_rng(100 + len(name))
    dy = rng.standard_normal((cfg.L, cfg.d))
    idx, gate, _ = O.route(cfg, h)
    g = O.backward(cfg, h, idx, gate, dy)[grad]
    base = h[name].astype(np.float64)
    for trial in range(3):
        v = rng.standard_normal(base.shape)
        eps = 1e-4 * max(1.0, float(np.abs(base).max()))
        hp, hm = dict(h), dict(h)
        hp[name] = (base + eps * v).astype(np.float32)
        hm[name] = (base - eps * v).astype(np.float32)
        lp, ip = _loss(cfg, hp, dy)
        lm, im = _loss(cfg, hm, dy)
        # the same selected sets (their order may swap where scores are close;
        # y does not depend on it)
        same = np.sort(idx, axis=1)
        assert np.array_equal(np.sort(ip, axis=1), same), "routing moved"
        assert np.array_equal(np.sort(im, axis=1), same), "routing moved"
        step = hp[name].astype(np.float64) - hm[name].astype(np.float64)
        pred = float(np.sum(g * step))
        fd = lp - lm
        scale = float(np.sum(np.abs(g * step))) + 1e-30
        assert abs(fd - pred) <= 2e-5 * scale, (name, trial, fd, pred)


def test_backward_of_a_single_token_and_expert_in_closed_form():
    """K = 1: the gate is 1 and its gradient vanishes, so the router receives
    nothing; y = SiLU(a) V[e] with a = x.W[e], hence dV[e] = SiLU(a) dy,
    dW[e] = (dy.V[e]) SiLU'(a) x, dx = (dy.V[e]) SiLU'(a) W[e], with
    SiLU'(a) = s(a)(1 + a(1 - s(a))) for the logistic s (scipy's expit)."""
    cfg = WL.Config("bwd-k1", L=1, d=6, Nr=3, Nc=2, k=1, K=1, B=1, dtype=WL.F32, seed=5)
    h = WL.make_inputs(cfg)
    idx, gate, _ = O.route(cfg, h)
    e = int(idx[0, 0])
    dy = np.arange(1.0, cfg.d + 1.0)[None, :] / 7.0
    r = O.backward(cfg, h, idx, gate, dy)
    x = h["x"][0].astype(np.float64)
    w = h["W"][e].astype(np.float64)
    v = h["V"][e].astype(np.float64)
    a = float(x @ w)
    sig = float(expit(a))
    s1 = sig * (1.0 + a * (1.0 - sig))
    sv = float(dy[0] @ v)
    np.testing.assert_allclose(r["dV"][e], a * sig * dy[0], rtol=1e-12)
    np.testing.assert_allclose(r["dW"][e], sv * s1 * x, rtol=1e-12)
    np.testing.assert_allclose(r["dx"][0], sv * s1 * w, rtol=1e-12, atol=1e-15)
    assert not np.delete(r["dW"], e, axis=0).any() and not np.delete(r["dV"], e, axis=0).any()
    assert np.all(np.abs(r["dWr"]) < 1e-15) and np.all(np.abs(r["dWc"]) < 1e-15)


def test_backward_invariants():
    """Softmax shift invariance: the bias gradients of each axis sum to zero;
    rows of experts no token chose get no gradient; the gradients are linear
    in dy."""
    cfg = BWD_CFGS[1]
    h = _bias_inputs(cfg)
    idx, gate, _ = O.route(cfg, h)
    rng = np.random.default_rng(7)
    dy1, dy2 = rng.standard_normal((2, cfg.L, cfg.d))
    r1 = O.backward(cfg, h, idx, gate, dy1)
    r2 = O.backward(cfg, h, idx, gate, dy2)
    r12 = O.backward(cfg, h, idx, gate, dy1 + 2.0 * dy2)
    for key in r1:
        np.testing.assert_allclose(r12[key], r1[key] + 2.0 * r2[key], rtol=1e-10, atol=1e-12)
    assert abs(r1["dbias_r"].sum()) < 1e-12 and abs(r1["dbias_c"].sum()) < 1e-12
    idle = np.setdiff1d(np.arange(cfg.N), idx)
    assert not r1["dW"][idle].any() and not r1["dV"][idle].any()
