"""Seeded synthetic inputs for the routed atomic-expert layer.

This module is shared by the oracle side (tests) and the CUDA side (tests,
bench) and holds none of the method's arithmetic: it only draws the inputs
(token activations ``x``, router matrices ``Wr``/``Wc``, expert matrices
``W``/``V`` and the optional Zipf logit bias) and rounds them to the storage
dtype.  Both sides receive byte-identical arrays.

Layouts (row-major):
  x  [L  x d]   token activations
  Wr [Nr x d]   row-router keys: row logit i of token t is x[t] . Wr[i]
  Wc [Nc x d]   column-router keys
  W  [N  x d]   input vectors w_in of the N = Nr*Nc atomic experts
  V  [N  x d]   output vectors w_out of the atomic experts
bf16 tensors are returned as uint16 arrays holding the raw bf16 bits
(round-to-nearest-even from an fp32 draw); fp32 tensors as float32.

Distributions: x ~ N(0, 1); Wr, Wc, W, V ~ N(0, 1/d).  Each tensor has its own
random stream (seed + a fixed tensor offset), and large tensors are drawn in
fixed chunks of CHUNK elements with one stream per chunk, so the bytes do not
depend on how many threads draw them.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 1 << 22  # elements per independent random stream

# fixed per-tensor stream offsets
_T_X, _T_WR, _T_WC, _T_W, _T_V, _T_PERM_R, _T_PERM_C = 0, 1, 2, 3, 4, 5, 6
_T_W1, _T_W2 = 7, 8  # the shared dense MLP
_T_U = 9  # the gate matrix of gated (SwiGLU) experts

F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    L: int
    d: int
    Nr: int
    Nc: int
    k: int
    K: int
    B: int
    dtype: int          # F32 or BF16
    seed: int = 0
    zipf_s: float = 0.0  # >0 adds the Zipf(s) log-weight bias to the router logits

    @property
    def N(self) -> int:
        return self.Nr * self.Nc

    @property
    def esize(self) -> int:
        return 4 if self.dtype == F32 else 2

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The five workloads of the routed layer (sizes as stated for the benchmark).
TINY = Config("tiny-fp32", L=128, d=64, Nr=64, Nc=64, k=8, K=8, B=32, dtype=F32)
BF16_16K = Config("bf16-N16K", L=4096, d=512, Nr=128, Nc=128, k=16, K=16, B=64, dtype=BF16)
SKEWED = Config("bf16-skewed-N256K", L=8192, d=1024, Nr=512, Nc=512, k=32, K=32, B=128,
                dtype=BF16, zipf_s=1.1)
PREFILL = Config("bf16-prefill-N1M", L=16384, d=2048, Nr=1024, Nc=1024, k=64, K=64, B=128,
                 dtype=BF16)
DECODE = Config("bf16-decode-N1M", L=64, d=2048, Nr=1024, Nc=1024, k=64, K=64, B=128,
                dtype=BF16)

CONFIGS = {c.name: c for c in (TINY, BF16_16K, SKEWED, PREFILL, DECODE)}

# A reduced prefill for counter captures: W, V 1 GiB each (far larger than L2),
# L*K = N (the same tasks per active expert as the prefill workload), and an
# fp32 accumulator above 40 MiB (the same execution path).
PREFILL_PROXY = Config("bf16-prefill-proxy-N256K", L=8192, d=2048, Nr=512, Nc=512, k=32, K=32,
                       B=128, dtype=BF16)
DECODE_PROXY = Config("bf16-decode-proxy-N256K", L=64, d=2048, Nr=512, Nc=512, k=64, K=64,
                      B=128, dtype=BF16)
EXTRA = {PREFILL_PROXY.name: PREFILL_PROXY, DECODE_PROXY.name: DECODE_PROXY}


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + (((u >> 16) & 1) + 0x7FFF)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (uint16) to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(seed: int, tensor: int, shape, scale: float, dtype: int) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16 if dtype == BF16 else np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def job(c: int) -> None:
        lo, hi = c * CHUNK, min(n, (c + 1) * CHUNK)
        rng = np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=(tensor, c)))
        buf = rng.standard_normal(hi - lo, dtype=np.float32)
        if scale != 1.0:
            buf *= np.float32(scale)
        out[lo:hi] = f32_to_bf16_bits(buf) if dtype == BF16 else buf

    if nchunks == 1:
        job(0)
    else:
        with ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            list(ex.map(job, range(nchunks)))
    return out.reshape(shape)


def zipf_bias(seed: int, tensor: int, n: int, s: float) -> np.ndarray:
    """Log Zipf(s) weights over a seeded random rank order: b[i] = -s*ln(1 + pi(i))."""
    rng = np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=(tensor, 0)))
    perm = rng.permutation(n)
    return (-s * np.log1p(perm.astype(np.float64))).astype(np.float32)


def make_inputs(cfg: Config, experts: bool = True) -> dict:
    """Draw the inputs of ``cfg``.  ``experts=False`` skips W and V (routing only)."""
    sc = 1.0 / np.sqrt(cfg.d)
    out = {
        "x": _normal(cfg.seed, _T_X, (cfg.L, cfg.d), 1.0, cfg.dtype),
        "Wr": _normal(cfg.seed, _T_WR, (cfg.Nr, cfg.d), sc, cfg.dtype),
        "Wc": _normal(cfg.seed, _T_WC, (cfg.Nc, cfg.d), sc, cfg.dtype),
        "bias_r": None,
        "bias_c": None,
    }
    if cfg.zipf_s > 0:
        out["bias_r"] = zipf_bias(cfg.seed, _T_PERM_R, cfg.Nr, cfg.zipf_s)
        out["bias_c"] = zipf_bias(cfg.seed, _T_PERM_C, cfg.Nc, cfg.zipf_s)
    if experts:
        out.update(make_experts(cfg))
    return out


def make_experts(cfg: Config) -> dict:
    """The expert matrices W, V [N x d] of ``cfg`` (they depend on seed, N, d, dtype only)."""
    sc = 1.0 / np.sqrt(cfg.d)
    return {"W": _normal(cfg.seed, _T_W, (cfg.N, cfg.d), sc, cfg.dtype),
            "V": _normal(cfg.seed, _T_V, (cfg.N, cfg.d), sc, cfg.dtype)}


def make_gate(cfg: Config) -> dict:
    """The gate matrix U [N x d] of gated (SwiGLU) experts, drawn like W
    (N(0, 1/d), so x.U[e] has unit scale)."""
    return {"U": _normal(cfg.seed, _T_U, (cfg.N, cfg.d), 1.0 / np.sqrt(cfg.d), cfg.dtype)}


def make_mlp(cfg: Config, F: int) -> dict:
    """Weights of a shared dense MLP of width F: W1 [F x d] ~ N(0, 1/d),
    W2 [d x F] ~ N(0, 1/F) (so both products keep unit scale)."""
    return {"W1": _normal(cfg.seed, _T_W1, (F, cfg.d), 1.0 / np.sqrt(cfg.d), cfg.dtype),
            "W2": _normal(cfg.seed, _T_W2, (cfg.d, F), 1.0 / np.sqrt(F), cfg.dtype)}


def sample_tokens(cfg: Config, n: int, seed: int = 1234) -> np.ndarray:
    """A seeded sorted subsample of token ids (all tokens when n >= L)."""
    if n >= cfg.L:
        return np.arange(cfg.L, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(cfg.L, size=n, replace=False)).astype(np.int64)


def random_routing(cfg: Config, seed: int = 99, pool: int = 4096) -> tuple:
    """A seeded routing decision for scheduler tests: idx [L, K] int32 with K
    distinct ids per token, about half of them drawn from a shared pool of
    ``pool`` ids (so groups hold several tokens and tokens share experts),
    and gate [L, K] float32 uniform in (0, 1]."""
    rng = np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=(cfg.L, cfg.K)))
    hot = rng.choice(cfg.N, size=min(pool, cfg.N), replace=False)
    idx = np.empty((cfg.L, cfg.K), np.int32)
    for t in range(cfg.L):
        n_hot = min(cfg.K // 2, len(hot))
        picks = set(rng.choice(hot, size=n_hot, replace=False).tolist())
        while len(picks) < cfg.K:
            picks.update(rng.integers(0, cfg.N, size=cfg.K - len(picks)).tolist())
        idx[t] = rng.permutation(np.fromiter(picks, np.int64, count=len(picks))[: cfg.K])
    gate = (1.0 - rng.random((cfg.L, cfg.K))).astype(np.float32)
    return idx, gate
