"""Mutation check of the oracle's pins.

Each mutant is a copy of ``oracle/oracle.c`` with one plausible mistake planted
in it: a flipped sign, a dropped term, a transposed operand, a wrong index, a
reversed tie-break, an off-by-one bound.  The copy is compiled with the
oracle's own flags, and the pin suite (``test_oracle_pins.py``, unchanged) runs
against it in a child process that loads it through ``OMNI_ORACLE_LIB``.  Every
mutant must make a pin fail.  The unmodified copy, built and run the same way,
must pass, so that a failure means the planted mistake and nothing else.

Every mutant keeps its memory accesses inside the oracle's buffers (ids stay
below N, rows below their counts), so a mutant fails by a wrong value, never by
a crash.  All of it runs on the CPU.
"""
import concurrent.futures as cf
import os
import re
import subprocess
import sys

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text of oracle.c, its replacement); each text occurs exactly once
MUTANTS = [
    # backward
    ("bwd-silu-grad-first-factor-only", "return sg * (1.0 + z * (1.0 - sg));", "return sg;"),
    ("bwd-softmax-drops-mean", "const double dS = gate[r * K + q] * (dg[q] - gdg);",
     "const double dS = gate[r * K + q] * dg[q];"),
    ("bwd-dV-without-gate", "dV[e * d + m] += gate[r * K + q] * h[r * K + q] * dym;",
     "dV[e * d + m] += h[r * K + q] * dym;"),
    ("bwd-da-without-gate", "da[r * K + q] = gate[r * K + q] * sk * silu_grad(a);",
     "da[r * K + q] = sk * silu_grad(a);"),
    ("bwd-dx-through-V", "for (int64_t m = 0; m < d; ++m) dxr[m] += da[r * K + q] * wrow[m];",
     "for (int64_t m = 0; m < d; ++m) dxr[m] += da[r * K + q] * vrow[m];"),
    ("bwd-column-of-row-index", "dlc[e % Nc] += dS;", "dlc[e / Nr % Nc] += dS;"),
    ("bwd-dWr-times-dy", "for (int64_t i = 0; i < Nr; ++i) dWr[i * d + m] += dzr[r * Nr + i] * xm;",
     "for (int64_t i = 0; i < Nr; ++i) dWr[i * d + m] += dzr[r * Nr + i] * dym;"),
    ("bwd-router-dx-dropped",
     "for (int64_t m = 0; m < d; ++m) dxr[m] += dlc[j] * wrow[m];",
     "for (int64_t m = 0; m < d; ++m) dxr[m] += 0.0 * wrow[m];"),
    ("bwd-bias-c-from-row-axis", "for (int64_t j = 0; j < Nc; ++j) dbc[j] += dzc[r * Nc + j];",
     "for (int64_t j = 0; j < Nc; ++j) dbc[j] += dzr[r * Nr + j % Nr];"),
    # shared dense MLP branch
    ("mlp-silu-on-the-output", "y[r * d + j] = dot(h, w2, F);",
     "y[r * d + j] = silu(dot(h, w2, F));"),
    ("mlp-w2-transposed", "load_row(W2, D->dtype, j, F, w2);",
     "for (int64_t f = 0; f < F; ++f) w2[f] = elem(W2, D->dtype, f * d + j);"),
    ("mlp-drops-last-hidden-unit", "h[f] = silu(dot(xt, w1, d));",
     "h[f] = f + 1 < F ? silu(dot(xt, w1, d)) : 0.0;"),
    ("mlp-linear-hidden", "h[f] = silu(dot(xt, w1, d));", "h[f] = dot(xt, w1, d);"),
    ("mlp-x-of-row-not-token", "load_row(x, D->dtype, tok[r], d, xt);",
     "load_row(x, D->dtype, r, d, xt);"),
    # atomic expert: sigma, dot product, operand rows
    ("silu-sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("dot-drops-last-term", "for (int64_t m = 0; m < n; ++m) s += a[m] * b[m];",
     "for (int64_t m = 0; m + 1 < n; ++m) s += a[m] * b[m];"),
    ("bf16-widening-shift", "((const uint16_t*)p)[i]) << 16", "((const uint16_t*)p)[i]) << 15"),
    ("bf16-drops-low-mantissa-bit", "((uint32_t)((const uint16_t*)p)[i]) << 16",
     "((uint32_t)(((const uint16_t*)p)[i] & 0xFFFEu)) << 16"),
    # router projections
    ("router-bias-dropped", "z[i] = dot(xrow, wrow, d) + (bias ? (double)bias[i] : 0.0);",
     "z[i] = dot(xrow, wrow, d);"),
    ("router-bias-sign", "z[i] = dot(xrow, wrow, d) + (bias ? (double)bias[i] : 0.0);",
     "z[i] = dot(xrow, wrow, d) - (bias ? (double)bias[i] : 0.0);"),
    ("router-x-of-token-0", "load_row(x, dtype, t, d, xrow);", "load_row(x, dtype, 0, d, xrow);"),
    ("router-matrix-transposed", "load_row(Wa, dtype, i, d, wrow);",
     "for (int64_t m = 0; m < d; ++m) wrow[m] = elem(Wa, dtype, m * n_axis + i);"),
    # per-axis log-softmax
    ("log-softmax-subtracts-max", "for (int64_t i = 0; i < n; ++i) z[i] -= lse;",
     "for (int64_t i = 0; i < n; ++i) z[i] -= mx;"),
    ("log-sum-exp-drops-max", "double lse = mx + log(s);", "double lse = log(s);"),
    ("log-softmax-rows-stride", "for (int64_t r = 0; r < rows; ++r) log_softmax(z + r * n, n);",
     "for (int64_t r = 0; r < rows; ++r) log_softmax(z + r, n);"),
    # orderings and the k x k merge
    ("order-ascending", "if (a->v > b->v) return -1;\n  if (a->v < b->v) return 1;",
     "if (a->v < b->v) return -1;\n  if (a->v > b->v) return 1;"),
    ("tie-break-larger-id", "return (a->id < b->id) ? -1 : (a->id > b->id);",
     "return (a->id > b->id) ? -1 : (a->id < b->id);"),
    ("expert-id-transposed", "tmp[c].id = ri[a] * Nc + ci[b];", "tmp[c].id = ci[b] * Nr + ri[a];"),
    ("joint-score-wrong-index", "tmp[c].v = rv[a] + cv[b];", "tmp[c].v = rv[a] + cv[a];"),
    ("merge-skips-last-row",
     "for (int64_t a = 0; a < k; ++a)\n        for (int64_t b = 0; b < k; ++b)",
     "for (int64_t a = 0; a + 1 < k; ++a)\n        for (int64_t b = 0; b < k; ++b)"),
    ("bruteforce-id-mapping", "s.v = lr[r * Nr + e / Nc] + lc[r * Nc + e % Nc];",
     "s.v = lr[r * Nr + e % Nr] + lc[r * Nc + e / Nr];"),
    ("bruteforce-next-is-Kth", "next[r] = (K < N) ? best[K].v : -INFINITY;",
     "next[r] = (K < N) ? best[K - 1].v : -INFINITY;"),
    # gate
    ("gate-numerator-unshifted", "gate[r * K + q] = exp(tmp[q].v - mx) / s;",
     "gate[r * K + q] = exp(tmp[q].v) / s;"),
    ("gate-sum-skips-first", "for (int64_t q = 0; q < K; ++q) s += exp(tmp[q].v - mx);",
     "for (int64_t q = 1; q < K; ++q) s += exp(tmp[q].v - mx);"),
    # scheduling
    ("group-of-rank-mod", "p->g = pos[p->e] / B;", "p->g = pos[p->e] % B;"),
    ("group-count-floor", "const int64_t G = (nu + B - 1) / B;", "const int64_t G = nu / B;"),
    ("sort-token-before-group",
     "if (a->g != b->g) return (a->g < b->g) ? -1 : 1;\n  if (a->t != b->t) return (a->t < b->t) ? -1 : 1;",
     "if (a->t != b->t) return (a->t < b->t) ? -1 : 1;\n  if (a->g != b->g) return (a->g < b->g) ? -1 : 1;"),
    ("cell-order-expert-desc", "return (a->e < b->e) ? -1 : (a->e > b->e);",
     "return (a->e > b->e) ? -1 : (a->e < b->e);"),
    ("group-offsets-off-by-one", "while (q < M && ts[q].g < g) ++q;",
     "while (q < M && ts[q].g <= g) ++q;"),
    # execution
    ("expert-order-drops-gate", "c[q] = task_gate[q] * silu(dot(xrow, wg + j * d, d));",
     "c[q] = silu(dot(xrow, wg + j * d, d));"),
    ("token-order-drops-gate", "double cq = gate[r * K + q] * silu(dot(xrow, wrow, d));",
     "double cq = silu(dot(xrow, wrow, d));"),
    ("slot-search-off-by-one", "if (uniq[u0 + mid] < e)", "if (uniq[u0 + mid] <= e)"),
    ("expert-order-V-row-of-first-expert", "elem(V, D->dtype, (int64_t)uniq[u0 + j] * d + m)",
     "elem(V, D->dtype, (int64_t)uniq[u0] * d + m)"),
    ("expert-order-overwrites-y", "yr[m] += c[q] * vg[j * w + (m - c0)];",
     "yr[m] = c[q] * vg[j * w + (m - c0)];"),
    # gated (SwiGLU) expert
    ("glu-drops-the-gate-factor", "if (U) c[q] *= dot(xrow, ug + j * d, d);", "if (U) c[q] *= 1.0;"),
    ("glu-gate-row-of-W", "if (U) c[q] *= dot(xrow, ug + j * d, d);",
     "if (U) c[q] *= dot(xrow, wg + j * d, d);"),
    ("glu-token-order-gate-of-first-expert", "load_row(U, D->dtype, e, d, urow);",
     "load_row(U, D->dtype, idx[r * K], d, urow);"),
    ("token-order-swaps-W-and-V",
     "load_row(W, D->dtype, e, d, wrow);\n        load_row(V, D->dtype, e, d, vrow);",
     "load_row(V, D->dtype, e, d, wrow);\n        load_row(W, D->dtype, e, d, vrow);"),
    ("token-order-x-of-row-not-token", "load_row(x, D->dtype, tok[r], d, xrow);",
     "load_row(x, D->dtype, r, d, xrow);"),
    ("expert-order-column-split-gap", "c1 = d * (tid + 1) / nth, w = c1 - c0;",
     "c1 = d * (tid + 1) / nth - 1, w = c1 - c0;"),
    ("traffic-counts-tasks", "wloaded += nb;", "wloaded += group_off[g + 1] - group_off[g];"),
]


def _workers():
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        cores = os.cpu_count() or 1
    jobs = max(1, min(4, cores // 2))
    return jobs, max(1, cores // jobs)


def _run_pins(lib_path, threads):
    env = dict(os.environ, OMNI_ORACLE_LIB=lib_path, OMP_NUM_THREADS=str(threads))
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    failed = re.findall(r"^FAILED (\S+)", r.stdout, flags=re.M)
    return r.returncode, (failed[0].split("::")[-1] if failed else r.stdout[-1500:])


def _mutant(tmp, src, name, old, new, threads):
    d = os.path.join(tmp, name)
    os.makedirs(d)
    c_path, so_path = os.path.join(d, "oracle.c"), os.path.join(d, "liboracle.so")
    with open(c_path, "w") as fh:
        fh.write(src if old is None else src.replace(old, new))
    oracle_build.compile_source(c_path, so_path, quiet=True)
    return _run_pins(so_path, threads)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(oracle_build.SRC) as fh:
        src = fh.read()
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"mutant {name}: its text no longer occurs once in oracle.c"
        assert old != new
    jobs, threads = _workers()
    with cf.ThreadPoolExecutor(jobs) as ex:
        control = ex.submit(_mutant, str(tmp_path), src, "unmodified", None, None, threads)
        futs = {name: ex.submit(_mutant, str(tmp_path), src, name, old, new, threads)
                for name, old, new in MUTANTS}
        results = {name: f.result() for name, f in futs.items()}
        rc0, out0 = control.result()
    assert rc0 == 0, f"the unmodified copy fails the pins:\n{out0}"
    survivors = {n: r for n, r in results.items() if r[0] != 1}
    assert not survivors, "mutants no pin catches (name: exit code, output):\n" + "\n".join(
        f"{n}: {rc}, {out}" for n, (rc, out) in survivors.items())
