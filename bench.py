"""Benchmark of the routed atomic-expert layer (Cartesian router -> expert-centric
schedule -> grouped execution) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload bf16-prefill-N1M|bf16-decode-N1M|...]

One step = one omni_moe_forward over a batch of L tokens of synthetic inputs
already resident in HBM.  L2 is flushed (a write larger than L2) before every
timed step, outside the step's CUDA events.  Prints one JSON line on rank 0.

Multi-GPU (torchrun): tokens are independent, so every rank runs its own
batch (its own x, replicated router and expert weights) with no collective on
the data path; value = all ranks' tokens / the slowest rank's time
(weak scaling).  --impl reference times the fp64 CPU oracle instead (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = "routed-layer tokens/s at N=1M,d=2048 (L=16K & L=64); % of TC/HBM roofline"
PRIMARY = WL.PREFILL
SECONDARY = WL.DECODE


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(
            j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def layer_work(cfg, n_active):
    """Algorithmic flops and bytes of one layer pass (the method's own work)."""
    e = cfg.esize
    flops = 2 * cfg.d * (cfg.Nr + cfg.Nc) * cfg.L + 4 * cfg.d * cfg.L * cfg.K
    bytes_ = (cfg.L * cfg.d * e + (cfg.Nr + cfg.Nc) * cfg.d * e + 2 * cfg.d * n_active * e
              + cfg.L * cfg.d * e)
    return flops, bytes_


def traffic_model(cfg, n_active):
    """The pages' parameter-traffic model of the two execution orders for one
    batch: token-centric D = 2d*L*K, expert-centric D = 2d*|E_active| (in
    bytes of the storage type), and the expert usage |E_active| / N."""
    e = cfg.esize
    d_tok = 2 * cfg.d * cfg.L * cfg.K * e
    d_exp = 2 * cfg.d * n_active * e
    return {"expert_usage": n_active / cfg.N, "tasks_per_active_expert": cfg.L * cfg.K / n_active
            if n_active else None, "d_token_centric_bytes": d_tok,
            "d_expert_centric_bytes": d_exp, "saving": d_tok / d_exp if d_exp else None}


def group_stats(group_off, B, n_active):
    """Tasks per group of a schedule, from its group offsets (int array of
    n_groups + 1 entries): count, min / median / mean / max, and the number of
    experts in the last group (the others hold B)."""
    go = np.asarray(group_off, dtype=np.int64)
    per = np.diff(go)
    if per.size == 0:
        return {"groups": 0}
    return {"groups": int(per.size), "tasks_min": int(per.min()),
            "tasks_median": float(np.median(per)), "tasks_mean": float(per.mean()),
            "tasks_max": int(per.max()), "experts_in_last_group": int(n_active - B * (per.size - 1))}


def group_density(task_token, group_off, B, n_active, block=128):
    """How dense each group's token x expert tile is: tasks_g / (T_g * B_g)
    with T_g the group's distinct tokens and B_g its experts (B, fewer in the
    last group), and the tasks per touched tile of `block` consecutive
    tokens by the group's B experts -- the fill of the tiles a dense
    (tensor-core) formulation of the grouped contraction would compute.
    task_token: the schedule's task tokens (sorted by token inside a group)."""
    tt = np.asarray(task_token, dtype=np.int64)
    go = np.asarray(group_off, dtype=np.int64)
    G = go.size - 1
    if G < 1:
        return {}
    dens, per_tile = [], []
    for g in range(G):
        t = tt[go[g]:go[g + 1]]
        if t.size == 0:
            continue
        bg = B if g < G - 1 else int(n_active - B * (G - 1))
        tokens = 1 + int(np.count_nonzero(np.diff(t)))
        tiles = 1 + int(np.count_nonzero(np.diff(t // block)))
        dens.append(t.size / (tokens * bg))
        per_tile.append(t.size / tiles)
    dens, per_tile = np.array(dens), np.array(per_tile)
    return {"density_median": float(np.median(dens)), "density_max": float(dens.max()),
            "tasks_per_tile_median": float(np.median(per_tile)),
            "tasks_per_tile_max": float(per_tile.max()), "tile_tokens": block}


# A synthetic batch whose groups are dense: 8192 tokens routed to 256
# experts (two groups of 128), for the timing of the tensor-core activations.
DENSE_SYNTH = WL.Config("bf16-dense-groups-N256", L=8192, d=1024, Nr=16, Nc=16, k=8, K=8, B=128,
                        dtype=WL.BF16, seed=0)


def expert_stage_bytes(cfg, n_active):
    """Algorithmic bytes of the grouped execution: active rows of W and V once,
    x read, y written."""
    e = cfg.esize
    return 2 * cfg.d * n_active * e + 2 * cfg.L * cfg.d * e


# DRAM bytes (read + write) of one expert-stage call, summed over its kernels,
# from ncu. The full-size stage is too large for a full capture; these values
# come from one capture per kernel of the bf16-prefill-proxy-N256K workload
# (1721.3 MB per stage call) scaled by the stage's algorithmic bytes (x3.90).
# Update them whenever the stage's kernels change, else report None.
STAGE_TRAFFIC = {
    "bf16-prefill-N1M": (6.713e9, "ncu dram__bytes of bf16-prefill-proxy-N256K, one capture per "
                                  "kernel (k_wsort_x, k_act, 2 x k_acc, 2 x k_slice_finish), "
                                  "scaled x3.90 by algorithmic bytes"),
}


def rank_inputs(cfg, rank):
    """Host inputs of one data-parallel rank: its own token batch x (seed +
    1000*rank for ranks > 0) with the shared router weights and biases."""
    host = WL.make_inputs(cfg, experts=False)
    if rank > 0:
        host["x"] = WL.make_inputs(cfg.with_(seed=cfg.seed + 1000 * rank), experts=False)["x"]
    return host


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks: a job step takes as long as its
    slowest rank (x itself with one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms):
    """Whole-job tokens/s: every rank processes its own batch in ms (max over ranks)."""
    return world * tokens_per_rank / (ms * 1e-3)


def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (the forward's own launches; memset
    nodes excluded), or None when the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kernels = 0
        for node in nodes[:n]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if err == rt.cudaError_t.cudaSuccess and kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kernels += 1
        return kernels
    except Exception:  # noqa: BLE001 -- introspection is best effort
        return None


class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle arm


def oracle_timing(cfg, target_s=10.0, max_tokens=None, h=None):
    """Time the fp64 oracle (route -> schedule -> expert-centric execution) on a
    bounded token sample sized for about target_s of CPU work.  Returns
    (tokens/s, sample tokens, seconds, threads, inputs); h: the inputs, when
    already drawn."""
    import oracle as O

    if h is None:
        h = WL.make_inputs(cfg)
    n = 64
    while True:
        tok = WL.sample_tokens(cfg, n)
        cs = cfg.with_(L=len(tok))
        hs = dict(h, x=np.ascontiguousarray(h["x"][tok]))
        t0 = time.perf_counter()
        O.moe_forward(cs, hs)
        dt = time.perf_counter() - t0
        if dt >= target_s or n >= cfg.L or (max_tokens and n >= max_tokens):
            return len(tok) / dt, len(tok), dt, O.num_threads(), h
        n = min(cfg.L, max(n * 2, int(n * target_s / max(dt, 1e-3) * 1.1)))
        if max_tokens:
            n = min(n, max_tokens)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = {**WL.CONFIGS, **WL.EXTRA}[args.workload]
    rate, n, dt, threads, _ = oracle_timing(cfg, target_s=max(2.0, 60.0 / max(1, args.steps)))
    # steps: repeat the bounded sample K times after W warm-ups (each a full pass)
    import oracle as O
    h = WL.make_inputs(cfg)
    tok = WL.sample_tokens(cfg, n)
    cs = cfg.with_(L=len(tok))
    hs = dict(h, x=np.ascontiguousarray(h["x"][tok]))
    for _ in range(args.warmup):
        O.moe_forward(cs, hs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.moe_forward(cs, hs)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = len(tok) / dt
    cpu = {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{len(tok)} of {cfg.L} tokens of {cfg.name} per step (route+schedule+"
                     "expert-centric execution, fp64)"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "L": cfg.L, "d": cfg.d, "Nr": cfg.Nr, "Nc": cfg.Nc,
                       "k": cfg.k, "K": cfg.K, "B": cfg.B, "sample_tokens": len(tok)},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm


def run_ours(args):
    import torch
    import torch.distributed as dist

    import atomic_expert_routing_b200 as omni
    import atomic_expert_routing_b200.sharded as omni_sharded
    from atomic_expert_routing_b200 import build as libbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    libbuild.build()
    hbm, tc, tc_sus, peak_src = measured_peaks()

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    cfg = {**WL.CONFIGS, **WL.EXTRA}[args.workload]
    host = rank_inputs(cfg, rank)  # own token batch per rank; weights are shared
    experts = WL.make_experts(cfg)
    d = {k: to_dev(v) for k, v in host.items()}
    d.update({k: to_dev(v) for k, v in experts.items()})
    del experts
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def measure(c, dd, steps, warmup, graph=True):
        D = omni.LayerDims.of(c)
        ws = omni.Workspace()
        counts = omni.new_counts(device)
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        stream = torch.cuda.Stream(device)

        def fwd():
            omni.moe_forward(D, dd["x"], dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                             dd["bias_c"], y=y, counts=counts, ws=ws, stream=stream)

        with torch.cuda.stream(stream):
            fwd()  # sizes the workspace
        torch.cuda.synchronize()
        g = None
        kernels = None
        if graph:
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g, stream=stream):
                fwd()
            kernels = graph_kernel_nodes(g)
            g.instantiate()
        run = g.replay if g is not None else fwd
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                flush.zero_()
                run()
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        with Clocks(local) as clk:
            t_wait = time.time()
            while not clk.lines and time.time() - t_wait < 3.0:
                time.sleep(0.01)
            barrier()
            with torch.cuda.stream(stream):
                for a, b in ev:
                    flush.zero_()
                    a.record(stream)
                    run()
                    b.record(stream)
            barrier()
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        torch.cuda.synchronize()
        n_active = int(counts[0].item())
        status = int(counts[2].item())
        return ms, n_active, status, clk.summary(), y, kernels

    def measure_expert_stage(c, dd, steps):
        """Grouped execution alone (its own events), for the kernel roofline."""
        D = omni.LayerDims.of(c)
        idx, gate, _ = omni.route(D, dd["x"], dd["Wr"], dd["Wc"], dd["bias_r"], dd["bias_c"])
        s = omni.schedule(D, idx, gate)
        ws = omni.Workspace()
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        stream = torch.cuda.current_stream(device)
        omni.expert_forward(D, dd["x"], dd["W"], dd["V"], s, y=y, ws=ws)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            omni.expert_forward(D, dd["x"], dd["W"], dd["V"], s, y=y, ws=ws)
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / steps, int(s["counts"][0].item())

    def measure_stages(c, dd, steps):
        """The three stages as separate calls with events between them (same
        kernels as the fused call), L2 flushed before each pass."""
        D = omni.LayerDims.of(c)
        stream = torch.cuda.current_stream(device)
        wr, wsd, we = omni.Workspace(), omni.Workspace(), omni.Workspace()
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        counts = omni.new_counts(device)

        def one(evs=None):
            if evs:
                evs[0].record(stream)
            idx, gate, _ = omni.route(D, dd["x"], dd["Wr"], dd["Wc"], dd["bias_r"], dd["bias_c"],
                                      ws=wr, with_score=False, counts=counts)
            if evs:
                evs[1].record(stream)
            s = omni.schedule(D, idx, gate, ws=wsd, counts=counts)
            if evs:
                evs[2].record(stream)
            omni.expert_forward(D, dd["x"], dd["W"], dd["V"], s, y=y, ws=we)
            if evs:
                evs[3].record(stream)
            return s

        s = one()
        torch.cuda.synchronize()
        tot = [0.0, 0.0, 0.0]
        for _ in range(steps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            flush.zero_()
            s = one(evs)
            torch.cuda.synchronize()
            for i in range(3):
                tot[i] += evs[i].elapsed_time(evs[i + 1])
        out = {"route": tot[0] / steps, "schedule": tot[1] / steps, "expert": tot[2] / steps}
        try:  # a diagnostic: it may not cost the line
            na, ng = (int(v) for v in counts[:2].cpu().tolist())
            go = s["group_off"][: ng + 1].cpu().numpy()
            out["groups"] = group_stats(go, c.B, na)
            out["groups"].update(group_density(s["task_token"].cpu().numpy(), go, c.B, na))
        except Exception as exc:  # noqa: BLE001
            out["groups"] = {"error": repr(exc)[:200]}
        return out

    def measure_ablation(c, dd, steps):
        """The pages' comparison on the same routing: expert-centric execution
        (schedule + grouped execution) against token-centric execution, each
        pass timed with events after an L2 flush."""
        D = omni.LayerDims.of(c)
        stream = torch.cuda.current_stream(device)
        idx, gate, _ = omni.route(D, dd["x"], dd["Wr"], dd["Wc"], dd["bias_r"], dd["bias_c"],
                                  with_score=False)
        wsd, we = omni.Workspace(), omni.Workspace()
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        counts = omni.new_counts(device)

        def ec():
            s = omni.schedule(D, idx, gate, ws=wsd, counts=counts)
            omni.expert_forward(D, dd["x"], dd["W"], dd["V"], s, y=y, ws=we)

        def tc_():
            omni.token_centric_forward(D, dd["x"], dd["W"], dd["V"], idx, gate, y=y,
                                       counts=counts)

        out = {}
        for name, fn in (("expert_centric_ms", ec), ("token_centric_ms", tc_)):
            fn()
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(steps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                tot += a.elapsed_time(b)
            out[name] = tot / steps
        out["token_over_expert"] = out["token_centric_ms"] / out["expert_centric_ms"]
        return out

    def measure_e2e(c, dd, steps, warmup):
        """The public call with host buffers: every step copies its x from pinned
        host memory to the device, runs the forward and copies its y back to
        pinned host memory.  Returns (serial ms, pipelined ms, H2D bytes, D2H
        bytes) per step.

        Serial: copy in, forward, copy out on one stream, one step at a time.
        Pipelined (double buffers, three streams): the copy-in of step i+1 and
        the copy-out of step i-1 run while step i computes, as a serving loop
        would; the L2 flush of each step runs on the compute stream inside the
        timed region, and one pair of events spans all the steps, from the
        first copy in to the last copy out."""
        D = omni.LayerDims.of(c)
        xh = torch.empty((c.L, c.d), dtype=D.torch_dtype).pin_memory()
        xh.copy_(dd["x"].cpu())
        yh = [torch.empty((c.L, c.d), dtype=D.torch_dtype).pin_memory() for _ in range(2)]
        xd = [torch.empty_like(dd["x"]) for _ in range(2)]
        y = [torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device) for _ in range(2)]
        counts = omni.new_counts(device)
        ws = omni.Workspace()
        comp, h2d, d2h = (torch.cuda.Stream(device) for _ in range(3))

        def fwd(j):
            omni.moe_forward(D, xd[j], dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                             dd["bias_c"], y=y[j], counts=counts, ws=ws, stream=comp)

        def serial_step():
            xd[0].copy_(xh, non_blocking=True)
            fwd(0)
            yh[0].copy_(y[0], non_blocking=True)

        with torch.cuda.stream(comp):
            for _ in range(warmup):
                flush.zero_()
                serial_step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        with torch.cuda.stream(comp):
            for a, b in ev:
                flush.zero_()
                a.record(comp)
                serial_step()
                b.record(comp)
        torch.cuda.synchronize()
        serial_ms = sum(a.elapsed_time(b) for a, b in ev) / steps

        x_ready = [torch.cuda.Event() for _ in range(2)]
        x_free = [torch.cuda.Event() for _ in range(2)]
        y_ready = [torch.cuda.Event() for _ in range(2)]
        y_free = [torch.cuda.Event() for _ in range(2)]

        def pipeline(n):
            for i in range(n):
                j = i & 1
                if i >= 2:  # buffer j: step i-2 has read its x and its y has left
                    h2d.wait_event(x_free[j])
                    comp.wait_event(y_free[j])
                with torch.cuda.stream(h2d):
                    xd[j].copy_(xh, non_blocking=True)
                x_ready[j].record(h2d)
                comp.wait_event(x_ready[j])
                with torch.cuda.stream(comp):
                    flush.zero_()
                    fwd(j)
                x_free[j].record(comp)
                y_ready[j].record(comp)
                d2h.wait_event(y_ready[j])
                with torch.cuda.stream(d2h):
                    yh[j].copy_(y[j], non_blocking=True)
                y_free[j].record(d2h)

        pipeline(max(warmup, 2))
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(h2d)
        comp.wait_event(t0)
        d2h.wait_event(t0)
        pipeline(steps)
        t1.record(d2h)  # the last copy out follows every other operation of the steps
        torch.cuda.synchronize()
        pipe_ms = t0.elapsed_time(t1) / steps
        return serial_ms, pipe_ms, xh.numel() * xh.element_size(), yh[0].numel() * yh[0].element_size()

    def timed_graph(fn, steps, warmup=2):
        """Mean CUDA-event time of fn captured in a graph, L2 flushed before
        each replay."""
        stream = torch.cuda.Stream(device)
        with torch.cuda.stream(stream):
            fn(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn(stream)
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                flush.zero_()
                g.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        with torch.cuda.stream(stream):
            for a, b in ev:
                flush.zero_()
                a.record(stream)
                g.replay()
                b.record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        del g
        return ms

    def measure_backward(c, dd, steps):
        """The backward of this batch (omni_moe_backward) on the forward's
        routing, gradients accumulated into fp32 arrays, timed alone after an
        L2 flush.  Algorithmic bytes: x and dy read; the active rows of W and
        V read and of dW and dV read and written in fp32; dx written in fp32;
        the router weights read and their fp32 gradients read and written;
        the routing read."""
        D = omni.LayerDims.of(c)
        idx = torch.empty((c.L, c.K), dtype=torch.int32, device=device)
        gate = torch.empty((c.L, c.K), dtype=torch.float32, device=device)
        counts = omni.new_counts(device)
        omni.moe_forward(D, dd["x"], dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                         dd["bias_c"], idx=idx, gate=gate, counts=counts)
        gen = torch.Generator(device=device)
        gen.manual_seed(c.seed + 91)
        dy = torch.randn((c.L, c.d), generator=gen, device=device).to(D.torch_dtype)
        f32 = torch.float32
        grads = {"dx": torch.empty((c.L, c.d), dtype=f32, device=device),
                 "dW": torch.zeros((c.N, c.d), dtype=f32, device=device),
                 "dV": torch.zeros((c.N, c.d), dtype=f32, device=device),
                 "dWr": torch.zeros((c.Nr, c.d), dtype=f32, device=device),
                 "dWc": torch.zeros((c.Nc, c.d), dtype=f32, device=device),
                 "dbias_r": torch.zeros(c.Nr, dtype=f32, device=device),
                 "dbias_c": torch.zeros(c.Nc, dtype=f32, device=device)}
        ws = omni.Workspace()

        def run(accumulate):
            def fwd(stream):
                omni.moe_backward(D, dd["x"], dd["Wr"], dd["Wc"], dd["W"], dd["V"], idx, gate,
                                  dy, grads=grads, accumulate=accumulate, counts=counts, ws=ws,
                                  stream=stream)
            return timed_graph(fwd, steps)

        ms = run(True)
        ms_over = run(False)
        na = int(counts[0].item())
        e = c.esize
        bytes_ = (2 * c.L * c.d * e + 2 * c.d * na * e + 2 * 2 * c.d * na * 4 + c.L * c.d * 4
                  + (c.Nr + c.Nc) * c.d * e + 2 * (c.Nr + c.Nc) * c.d * 4 + 8 * c.L * c.K)
        flops = 4 * c.L * (c.Nr + c.Nc) * c.d + 8 * c.L * c.K * c.d
        del grads, ws, dy
        torch.cuda.empty_cache()
        # overwriting skips the reads of the old gradient rows
        bytes_over = bytes_ - 2 * c.d * na * 4 - (c.Nr + c.Nc) * c.d * 4
        return {"ms": ms, "n_active": na, "tokens_per_s": c.L / (ms * 1e-3),
                "roofline": {"bound": "hbm", "bytes": bytes_, "flops": flops,
                             "achieved": bytes_ / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                             "frac": bytes_ / (hbm * 1e9) / (ms * 1e-3), "peak_src": peak_src},
                "overwrite": {"ms": ms_over, "bytes": bytes_over,
                              "frac": bytes_over / (hbm * 1e9) / (ms_over * 1e-3)},
                "note": "gradients accumulated into fp32 arrays (accumulate); overwrite: the "
                        "first micro-batch, old gradient rows not read"}

    if args.backward_only:
        # profiling entry: the backward of this workload alone (no JSON line)
        rec = measure_backward(cfg, d, args.steps)
        if rank == 0:
            print(f"backward {cfg.name}: {rec['ms']:.4f} ms, {rec['roofline']['frac']:.3f} of "
                  f"HBM; overwriting: {rec['overwrite']['ms']:.4f} ms, "
                  f"{rec['overwrite']['frac']:.3f}", flush=True)
        return 0
    ms, n_active, status, clocks, _, kernels = measure(cfg, d, args.steps, args.warmup)
    ms_all = max_over_ranks(ms, world, device)
    # a serving loop runs many steps: the unoverlapped first copy in and
    # last copy out (about 2.4 ms at prefill) are spread over at least 30
    e2e_steps = max(30, args.steps)
    e2e_serial_ms, e2e_ms, h2d, d2h = measure_e2e(cfg, d, e2e_steps, args.warmup)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, world, device)
    st_ms, n_act2 = measure_expert_stage(cfg, d, max(3, args.steps // 2))
    stages = measure_stages(cfg, d, max(3, args.steps // 2))
    sched_groups = stages.pop("groups", None)

    ablation = measure_ablation(cfg, d, max(3, args.steps // 2))

    def summary(sc, dd, steps, warmup, with_stages):
        ms2, na2, st2, _, _, _ = measure(sc, dd, steps, warmup)
        ms2 = max_over_ranks(ms2, world, device)
        f2, b2 = layer_work(sc, na2)
        rec = {"value": job_throughput(world, sc.L, ms2), "unit": "tokens/s", "ms_per_step": ms2,
               "n_active": na2, "device_status": st2,
               "layer_roofline": {"bound": "hbm" if b2 / (hbm * 1e9) > f2 / (tc * 1e12) else "tensor",
                                  "frac": max(f2 / (tc * 1e12), b2 / (hbm * 1e9)) / (ms2 * 1e-3),
                                  "bytes": b2, "flops": f2}}
        if with_stages:
            st2 = measure_stages(sc, dd, 10)
            rec["schedule_groups"] = st2.pop("groups", None)
            rec["stages_ms"] = st2
            rec["ablation"] = measure_ablation(sc, dd, 10)
        return rec

    def measure_mlp(c, dd, F, steps):
        """The shared dense MLP branch (omni_shared_mlp: two tcgen05 GEMMs) of
        width F on this batch, timed alone with events after an L2 flush;
        2 * 2 * L * d * F flops against the measured bf16 peak (burst)."""
        D = omni.LayerDims.of(c)
        w = {k: to_dev(v) for k, v in WL.make_mlp(c, F).items()}
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        ws = omni.Workspace()
        stream = torch.cuda.current_stream(device)
        for _ in range(3):
            omni.shared_mlp(D, dd["x"], w["W1"], w["W2"], y=y, ws=ws)
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            omni.shared_mlp(D, dd["x"], w["W1"], w["W2"], y=y, ws=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        ms = tot / steps
        flops = 4.0 * c.L * c.d * F
        ach = flops / (ms * 1e-3) / 1e12
        return {"F": F, "ms": ms, "kernel": "two tcgen05 GEMMs (SiLU epilogue to bf16 H; add into y)",
                "roofline": {"bound": "tensor", "achieved": ach, "peak": tc, "unit": "TFLOP/s",
                             "frac": ach / tc, "flops": flops, "peak_src": peak_src}}

    def measure_dense_paths(steps):
        """A batch routed to 256 experts by 8192 tokens (two groups, 512 tasks
        per touched 128-token tile): its grouped execution with the dense
        groups' activations on the tensor cores (OMNI_FLAG_DENSE_TENSOR_CORES)
        and with every activation on the CUDA cores (the default), each after
        an L2 flush."""
        dc = DENSE_SYNTH
        hs = WL.make_inputs(dc)
        ds = {k: to_dev(v) for k, v in hs.items()}
        out = {"workload": dc.name}
        for name, flags in (("tensor_cores", omni.OMNI_FLAG_DENSE_TENSOR_CORES), ("cuda_cores", 0)):
            D = omni.LayerDims.of(dc, flags=flags)
            idx, gate, _ = omni.route(D, ds["x"], ds["Wr"], ds["Wc"], with_score=False)
            counts = omni.new_counts(device)
            counts[3] = -1
            sch = omni.schedule(D, idx, gate, counts=counts)
            y = torch.empty((dc.L, dc.d), dtype=D.torch_dtype, device=device)
            ws = omni.Workspace()
            stream = torch.cuda.current_stream(device)
            for _ in range(3):
                omni.expert_forward(D, ds["x"], ds["W"], ds["V"], sch, y=y, ws=ws)
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(steps):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                omni.expert_forward(D, ds["x"], ds["W"], ds["V"], sch, y=y, ws=ws)
                e1.record(stream)
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1)
            out[name] = {"expert_ms": tot / steps, "dense_groups": int(counts[3].item()),
                         "groups": int(counts[1].item())}
        del ds
        torch.cuda.empty_cache()
        return out

    def measure_shards(c, dd, steps):
        """Expert-sharded forward on this batch, one G-way split at a time:
        every shard's per-process work (routing, schedule, its own experts'
        execution into an fp32 partial, the cast) timed alone on this GPU.
        The job's step is the slowest shard plus one all-reduce of the
        L x d fp32 partials, which one GPU cannot time: it is estimated from
        the measured 8-GPU all-reduce bus bandwidth, 725 GB/s."""
        D = omni.LayerDims.of(c)
        out = {"workload": c.name, "allreduce_busbw_gbs": 725.0,
               "note": "per-shard times measured; the all-reduce and all-gather times are "
                       "estimates; split_routing: each process routes L/G tokens and the "
                       "routing is all-gathered (sharded.forward_split_routing)"}
        part_bytes = c.L * c.d * 4
        # the batch's routing, for the shards that take it as input
        r_idx = torch.empty((c.L, c.K), dtype=torch.int32, device=device)
        r_gate = torch.empty((c.L, c.K), dtype=torch.float32, device=device)
        omni.moe_forward(D, dd["x"], dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                         dd["bias_c"], idx=r_idx, gate=r_gate)
        for G in (2, 4, 8):
            shard_ms, active, split_ms = [], [], []
            tok = omni_sharded.token_ranges(c.L, G)
            for lo, hi in omni_sharded.shard_ranges(c.N, G):
                ws = omni.Workspace()
                counts = omni.new_counts(device)
                yp = torch.empty((c.L, c.d), dtype=torch.float32, device=device)
                y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
                Wl, Vl = dd["W"][lo:hi], dd["V"][lo:hi]

                def fwd(stream):
                    omni.moe_forward_shard(D, dd["x"], dd["Wr"], dd["Wc"], Wl, Vl, lo, hi,
                                           dd["bias_r"], dd["bias_c"], y_part=yp, counts=counts,
                                           ws=ws, stream=stream)
                    omni.cast_output(D, yp, y=y, stream=stream)

                shard_ms.append(timed_graph(fwd, steps))
                active.append(int(counts[0].item()))
                # split routing: this process's L/G tokens routed, then its
                # experts executed from the whole routing
                g = len(split_ms)
                t0, t1 = tok[g]
                Dg = omni.LayerDims(t1 - t0, c.d, c.Nr, c.Nc, c.k, c.K, c.B, c.dtype, 0)
                ws_r = omni.Workspace()
                xg = dd["x"][t0:t1]
                i_g = torch.empty((t1 - t0, c.K), dtype=torch.int32, device=device)
                g_g = torch.empty((t1 - t0, c.K), dtype=torch.float32, device=device)
                c_g = omni.new_counts(device)

                def fwd_split(stream):
                    if t1 > t0:
                        omni.route(Dg, xg, dd["Wr"], dd["Wc"], dd["bias_r"], dd["bias_c"],
                                   counts=c_g, ws=ws_r, stream=stream, with_score=False,
                                   out=(i_g, g_g))
                    omni.moe_forward_shard_routed(D, dd["x"], Wl, Vl, lo, hi, r_idx, r_gate,
                                                  y_part=yp, counts=counts, ws=ws, stream=stream)
                    omni.cast_output(D, yp, y=y, stream=stream)

                split_ms.append(timed_graph(fwd_split, steps))
                del ws, yp, y, ws_r
            ar = part_bytes * 2 * (G - 1) / G / (725.0e9) * 1e3
            ag = c.L * c.K * 8 * (G - 1) / G / (725.0e9) * 1e3
            out[str(G)] = {"shard_ms": shard_ms, "max_shard_ms": max(shard_ms),
                           "active_per_shard": active, "allreduce_ms_estimate": ar,
                           "step_ms_estimate": max(shard_ms) + ar,
                           "split_routing_shard_ms": split_ms,
                           "allgather_ms_estimate": ag,
                           "split_routing_step_ms_estimate": max(split_ms) + ag + ar,
                           "expert_bytes_per_gpu": 2 * c.d * max(active) * c.esize}
        torch.cuda.empty_cache()
        return out

    def measure_glu(c, dd, steps):
        """The gated (SwiGLU) forward of this batch: a third expert matrix U,
        drawn on the device (timing only), read once per active expert."""
        D = omni.LayerDims.of(c)
        gen = torch.Generator(device=device)
        gen.manual_seed(c.seed + 77)
        U = (torch.randn((c.N, c.d), generator=gen, device=device, dtype=torch.float32)
             / np.sqrt(c.d)).to(D.torch_dtype)
        ws = omni.Workspace()
        counts = omni.new_counts(device)
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)

        def fwd(stream):
            omni.moe_forward(D, dd["x"], dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                             dd["bias_c"], U=U, y=y, counts=counts, ws=ws, stream=stream)

        ms = timed_graph(fwd, steps)
        na = int(counts[0].item())
        flops, bytes_ = layer_work(c, na)
        bytes_ += c.d * na * c.esize  # the U rows
        del U, ws
        torch.cuda.empty_cache()
        return {"ms_per_step": ms, "value": c.L / (ms * 1e-3), "unit": "tokens/s", "n_active": na,
                "layer_roofline": {"bound": "hbm", "frac": bytes_ / (hbm * 1e9) / (ms * 1e-3),
                                   "bytes": bytes_}}

    def measure_rotating_x(c, dd, steps, nbatch=8):
        """The forward of the workload with x rotated among nbatch seeded
        token batches (one graph per batch, replayed in turn), L2 flushed
        before each step as in the headline: a step never finds its x, or
        rows its tokens share with the previous batch, in L2."""
        D = omni.LayerDims.of(c)
        ws = omni.Workspace()
        counts = omni.new_counts(device)
        y = torch.empty((c.L, c.d), dtype=D.torch_dtype, device=device)
        xs = [dd["x"]] + [to_dev(rank_inputs(c.with_(seed=c.seed + 7919 * (b + 1)), rank)["x"])
                          for b in range(nbatch - 1)]
        stream = torch.cuda.Stream(device)
        graphs = []
        for xb in xs:
            def fwd(xb=xb):
                omni.moe_forward(D, xb, dd["Wr"], dd["Wc"], dd["W"], dd["V"], dd["bias_r"],
                                 dd["bias_c"], y=y, counts=counts, ws=ws, stream=stream)
            with torch.cuda.stream(stream):
                fwd()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fwd()
            graphs.append(g)
        with torch.cuda.stream(stream):
            for g in graphs:
                flush.zero_()
                g.replay()
        n = max(steps, nbatch)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        with torch.cuda.stream(stream):
            for j, (a, b) in enumerate(ev):
                flush.zero_()
                a.record(stream)
                graphs[j % nbatch].replay()
                b.record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in ev) / n
        del graphs, xs, ws
        torch.cuda.empty_cache()
        return {"ms_per_step": ms, "batches": nbatch, "steps": n,
                "value": job_throughput(world, c.L, ms), "unit": "tokens/s"}

    extra = {}
    if args.workload == PRIMARY.name and not args.no_secondary:
        if world == 1:
            # single-process extras (each rank of a group would repeat them):
            # the shared dense MLP of the same batch (width F = d), the
            # tensor-core dense groups, expert shards, gated experts, the
            # backward and the rotating-batch check
            extra["shared_mlp"] = measure_mlp(cfg, d, cfg.d, max(3, args.steps // 2))
            extra["dense_groups"] = measure_dense_paths(max(3, args.steps // 2))
            extra["expert_shards"] = measure_shards(cfg, d, 3)
            extra["glu"] = measure_glu(cfg, d, max(3, args.steps // 2))
            extra["backward"] = measure_backward(cfg, d, max(3, args.steps // 2))
            extra["rotating_x"] = measure_rotating_x(cfg, d, args.steps)
        sc = SECONDARY
        host2 = rank_inputs(sc, rank)
        d2 = dict(d, x=to_dev(host2["x"]), bias_r=None, bias_c=None)
        extra[sc.name] = summary(sc, d2, max(args.steps, 20), max(args.warmup, 5), True)
        # the decode batch through the public call with host buffers.  Its
        # copies are 256 KiB each way, so one step at a time (the L2 flush
        # outside the events) is the figure; the pipelined loop times its
        # 256 MiB flush inside every step, which is most of a decode step
        es, ep, eh, eo = measure_e2e(sc, d2, max(args.steps, 20), max(args.warmup, 5))
        extra[sc.name]["e2e"] = {"value": job_throughput(world, sc.L, es), "unit": "tokens/s",
                                 "ms_per_step": es, "h2d_bytes_per_step": eh,
                                 "d2h_bytes_per_step": eo,
                                 "mode": "serial: copy in, forward, copy out on one stream",
                                 "pipelined_with_flush": {"value": job_throughput(world, sc.L, ep),
                                                          "ms_per_step": ep}}
        del d2
        # the other workloads (parity configurations), each with its own weights
        for sc in (WL.TINY, WL.BF16_16K, WL.SKEWED):
            hs = rank_inputs(sc, rank)
            hs.update(WL.make_experts(sc))
            ds = {k: to_dev(v) for k, v in hs.items()}
            extra[sc.name] = summary(sc, ds, max(args.steps, 10), max(args.warmup, 3), True)
            del ds, hs
            torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    flops, bytes_ = layer_work(cfg, n_active)
    t_f = flops / (tc * 1e12)
    t_b = bytes_ / (hbm * 1e9)
    eb = expert_stage_bytes(cfg, n_act2)
    achieved = eb / (st_ms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, n, dt, threads, h_cpu = oracle_timing(cfg, target_s=args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} of {cfg.L} tokens of {cfg.name} (route+schedule+expert-centric "
                         f"execution, fp64), {dt:.1f} s"}
        # the same oracle on one thread, over a smaller sample
        import oracle as O
        try:
            O.set_num_threads(1)
            rate1, n1, dt1, _, _ = oracle_timing(cfg, target_s=min(2.0, args.cpu_seconds),
                                                 max_tokens=max(64, n // 8), h=h_cpu)
        finally:
            O.set_num_threads(threads)
        cpu["value_1_thread"] = rate1
        cpu["sample_1_thread"] = f"{n1} tokens, {dt1:.1f} s"
    line = {
        "metric": METRIC,
        "value": job_throughput(world, cfg.L, ms_all),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_all,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == WL.BF16 else "f32",
        "data": "synthetic",
        "config": {"workload": cfg.name, "L": cfg.L, "d": cfg.d, "Nr": cfg.Nr, "Nc": cfg.Nc,
                   "N": cfg.N, "k": cfg.k, "K": cfg.K, "B": cfg.B, "l2": "flushed before each step",
                   "graph": True, "parallelism": f"dp{world} (independent token batches)"},
        "n_active": n_active,
        "traffic_model": traffic_model(cfg, n_active),
        "device_status": status,
        "stages_ms": stages,
        "schedule_groups": sched_groups,
        "ablation": ablation,
        "layer_roofline": {"bound": "hbm" if t_b >= t_f else "tensor",
                           "frac": max(t_f, t_b) / (ms_all * 1e-3), "bytes": bytes_,
                           "flops": flops, "peak_src": peak_src},
        "roofline": {"kernel": "grouped expert-centric execution (omni_expert_forward)",
                     "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm,
                     "traffic": STAGE_TRAFFIC.get(cfg.name, (None, None))[0],
                     "traffic_src": STAGE_TRAFFIC.get(cfg.name, (None, None))[1],
                     "algorithmic_bytes": eb,
                     "ms": st_ms, "peak_src": peak_src},
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(world, cfg.L, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "mode": "pipelined: double buffers on three streams; the copy in of step i+1 "
                        "and the copy out of step i-1 overlap step i; L2 flush inside",
                "serial": {"value": job_throughput(world, cfg.L, e2e_serial_ms),
                           "ms_per_step": e2e_serial_ms}},
        # the library's kernels in the timed region: kernel nodes of the
        # captured forward (one replay per step)
        "gpu_launches": kernels * args.steps if kernels is not None else None,
        "kernels_per_step": kernels,
        "clocks": clocks,
    }
    if extra:
        line["also"] = extra
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=PRIMARY.name, choices=sorted(WL.CONFIGS) + sorted(WL.EXTRA))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward of the workload (profiling; no JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
