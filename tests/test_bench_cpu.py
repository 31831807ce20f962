"""The benchmark on the CPU.  Its reference arm (the fp64 oracle on the host
cores): the JSON line carries the contract's keys, at least 3 warm-up steps
run, and ranks other than 0 do no work.  Its roofline arithmetic, worked by
hand."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
        "tiny-fp32", "--steps", "2", "--warmup", "1"]


def _run(env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run(ARGS, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)


def test_reference_arm_prints_one_contract_line():
    r = _run()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    d = json.loads(lines[-1])
    assert d["impl"] == "reference"
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["n_gpus"] == 1
    assert d["warmup"] == 3  # fewer than 3 warm-up steps are raised to 3
    assert d["config"]["workload"] == "tiny-fp32"
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == d["value"] and cpu["cores"] >= 1
    assert cpu["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert abs(d["ms_per_step"] - d["config"]["sample_tokens"] / d["value"] * 1e3) < 1e-6 * d["ms_per_step"] + 1e-9


def test_reference_arm_other_ranks_exit_without_work():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def _golden_traffic():
    rows = {}
    with open(os.path.join(ROOT, "tests", "golden", "traffic_model.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                rows[k] = v
    return rows


def test_roofline_arithmetic():
    """The bench's algorithmic work, worked by hand at the prefill and decode
    sizes: F = 2d(Nr+Nc)L + 4dLK, layer bytes = x + Wr + Wc + 2d|E|esize + y,
    the expert stage's bytes = 2d|E|esize + x + y, and its parameter bytes are
    the pages' expert-centric traffic 2d|E_active| elements (golden file)."""
    import bench
    import workloads as WL

    p, n_act = WL.PREFILL, 652642
    f, b = bench.layer_work(p, n_act)
    assert f == 137_438_953_472 + 8_589_934_592 == 146_028_888_064
    x = y = 16384 * 2048 * 2                     # 64 MiB each, bf16
    keys = 2 * 1024 * 2048 * 2                   # Wr and Wc
    rows = 2 * 2048 * n_act * 2                  # W and V rows of the active experts
    assert b == x + keys + rows + y == 5_489_049_600
    assert bench.expert_stage_bytes(p, n_act) == rows + x + y == 5_480_660_992
    g = _golden_traffic()
    env = {"d": p.d, "L": p.L, "K": p.K, "n_active": n_act}
    assert eval(g["expert_centric"], {}, env) * p.esize == rows
    assert eval(g["token_centric"], {}, env) * p.esize == 2 * 2048 * 16384 * 64 * 2
    f, _ = bench.layer_work(WL.DECODE, 4082)
    assert f == 536_870_912 + 33_554_432 == 570_425_344
    assert bench.job_throughput(1, 16384, 1.6) == 16384 / 1.6e-3
    assert bench.job_throughput(4, 16384, 1.6) == 4 * 16384 / 1.6e-3


def test_traffic_model_of_the_pages():
    """Token-centric 2d*L*K against expert-centric 2d*|E_active| parameter
    traffic (golden formulas), in bytes, with the expert usage |E|/N."""
    import bench
    import workloads as WL

    p, n_act = WL.PREFILL, 652642
    t = bench.traffic_model(p, n_act)
    g = _golden_traffic()
    env = {"d": p.d, "L": p.L, "K": p.K, "n_active": n_act}
    assert t["d_token_centric_bytes"] == eval(g["token_centric"], {}, env) * 2 == 8_589_934_592
    assert t["d_expert_centric_bytes"] == eval(g["expert_centric"], {}, env) * 2 == 5_346_443_264
    assert abs(t["saving"] - 8_589_934_592 / 5_346_443_264) < 1e-12
    assert abs(t["expert_usage"] - n_act / 2 ** 20) < 1e-15
    assert abs(t["tasks_per_active_expert"] - 16384 * 64 / n_act) < 1e-12
    assert bench.traffic_model(WL.TINY, 0)["saving"] is None


def test_group_stats():
    """Tasks per group from group offsets, worked by hand."""
    import bench

    g = bench.group_stats([0, 5, 7, 16, 18], B=4, n_active=14)
    assert g == {"groups": 4, "tasks_min": 2, "tasks_median": 3.5, "tasks_mean": 4.5,
                 "tasks_max": 9, "experts_in_last_group": 2}
    assert bench.group_stats([0], B=4, n_active=0) == {"groups": 0}


def test_group_density_by_hand():
    """Two groups of B = 4 experts (n_active = 6: the last group has 2).
    Group 0: tokens 0, 0, 1, 200 (3 tokens; tiles of 128 tokens: 0 and 1) ->
    density 4 / (3 * 4), 4 / 2 tasks per touched tile.  Group 1: tokens 5, 5
    (1 token, 2 experts) -> density 2 / (1 * 2), 2 tasks in one tile."""
    import bench

    d = bench.group_density([0, 0, 1, 200, 5, 5], [0, 4, 6], B=4, n_active=6)
    assert abs(d["density_median"] - (4 / 12 + 1.0) / 2) < 1e-12
    assert d["density_max"] == 1.0
    assert d["tasks_per_tile_median"] == 2.0 and d["tasks_per_tile_max"] == 2.0
    assert bench.group_density([], [0], B=4, n_active=0) == {}
