"""The seeded input recipe shared by the oracle and the CUDA path.

x ~ N(0, 1); Wr, Wc, W, V ~ N(0, 1/d); each tensor from its own random
stream; the skewed workload's log Zipf(s) bias b[i] = -s ln(1 + pi(i)) over a
seeded permutation pi; token sub-samples and the scheduler tests' routing
decisions.  The bf16 rounding of the generator is pinned with the oracle's
pins.
"""
import numpy as np

import workloads as WL


def _f32(a, cfg):
    return WL.bf16_bits_to_f32(a) if cfg.dtype == WL.BF16 else a


def test_inputs_are_deterministic_and_streams_independent():
    cfg = WL.BF16_16K.with_(L=512)
    a = WL.make_inputs(cfg)
    b = WL.make_inputs(cfg)
    for k in ("x", "Wr", "Wc", "W", "V"):
        assert np.array_equal(a[k], b[k]), k
    # another seed changes every tensor; equal shapes never share a stream
    c = WL.make_inputs(cfg.with_(seed=cfg.seed + 1))
    for k in ("x", "Wr", "Wc", "W", "V"):
        assert not np.array_equal(a[k], c[k]), k
    assert not np.array_equal(a["Wr"], a["Wc"])  # Nr == Nc here
    assert not np.array_equal(a["W"], a["V"])
    # the routing tensors do not depend on whether the experts are drawn
    r = WL.make_inputs(cfg, experts=False)
    for k in ("x", "Wr", "Wc"):
        assert np.array_equal(a[k], r[k]), k
    assert "W" not in r


def test_input_distributions():
    """Sample moments within a few standard errors of N(0, 1) and N(0, 1/d)."""
    cfg = WL.BF16_16K.with_(L=2048)
    h = WL.make_inputs(cfg)
    for k, var in (("x", 1.0), ("Wr", 1.0 / cfg.d), ("Wc", 1.0 / cfg.d), ("W", 1.0 / cfg.d),
                   ("V", 1.0 / cfg.d)):
        v = _f32(h[k], cfg).astype(np.float64).ravel()
        n = v.size
        assert abs(v.mean()) < 6 * np.sqrt(var / n), k
        # var of the sample variance of a normal: 2 var^2 / n (+ bf16 rounding, 2^-9 relative)
        assert abs(v.var() / var - 1) < 6 * np.sqrt(2.0 / n) + 2e-3, k
        kurt = ((v - v.mean()) ** 4).mean() / v.var() ** 2
        assert abs(kurt - 3.0) < 0.1, k


def test_zipf_bias_is_a_permuted_log_zipf():
    """b[i] = -s ln(1 + pi(i)): as a multiset, -s ln(1 + r) for r = 0..n-1; the
    weights exp(b) are (1 + r)^-s, so the most favoured id has bias 0."""
    s, n = 1.1, 1024
    b = WL.zipf_bias(0, 5, n, s).astype(np.float64)
    want = -s * np.log1p(np.arange(n, dtype=np.float64))
    np.testing.assert_allclose(np.sort(b)[::-1], want, rtol=1e-6, atol=1e-6)
    w = np.exp(np.sort(b)[::-1])
    np.testing.assert_allclose(w, (1.0 + np.arange(n)) ** -s, rtol=1e-5)
    assert b.max() == 0.0 and np.count_nonzero(b == 0.0) == 1
    # seeded: same stream same order; another tensor key another order
    assert np.array_equal(WL.zipf_bias(0, 5, n, s), WL.zipf_bias(0, 5, n, s))
    assert not np.array_equal(WL.zipf_bias(0, 5, n, s), WL.zipf_bias(0, 6, n, s))
    # the skewed workload carries it on both axes; the others carry none
    h = WL.make_inputs(WL.SKEWED, experts=False)
    assert h["bias_r"].shape == (WL.SKEWED.Nr,) and h["bias_c"].shape == (WL.SKEWED.Nc,)
    assert WL.make_inputs(WL.TINY, experts=False)["bias_r"] is None


def test_sample_tokens():
    cfg = WL.BF16_16K
    t = WL.sample_tokens(cfg, 300)
    assert t.dtype == np.int64 and len(t) == 300
    assert np.all(np.diff(t) > 0) and t[0] >= 0 and t[-1] < cfg.L
    assert np.array_equal(t, WL.sample_tokens(cfg, 300))
    assert np.array_equal(WL.sample_tokens(cfg, cfg.L + 5), np.arange(cfg.L))


def test_random_routing_for_scheduler_tests():
    cfg = WL.Config("rr", L=300, d=8, Nr=64, Nc=32, k=16, K=16, B=8, dtype=WL.F32)
    idx, gate = WL.random_routing(cfg, pool=64)
    assert idx.shape == (cfg.L, cfg.K) and idx.dtype == np.int32
    assert idx.min() >= 0 and idx.max() < cfg.N
    assert all(len(set(r.tolist())) == cfg.K for r in idx)
    assert gate.dtype == np.float32 and gate.min() > 0 and gate.max() <= 1
    # the shared pool makes tokens share experts
    assert len(np.unique(idx)) < 0.5 * idx.size
    i2, g2 = WL.random_routing(cfg, pool=64)
    assert np.array_equal(idx, i2) and np.array_equal(gate, g2)
