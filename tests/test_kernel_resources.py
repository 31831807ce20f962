"""Register and spill budget of the kernels on the benchmarked paths, read from
the compiler's resource report (nvcc -Xptxas=-v, kept beside each object by
the build).  None of them may spill to local memory; the decode selection's
8-byte spill is the one recorded exception.  Runs on the CPU (nvcc
cross-compiles for sm_100a)."""
import os
import re
import subprocess

import pytest

from atomic_expert_routing_b200 import build as libbuild

# demangled-name prefix -> largest spill (bytes, stores + loads) allowed
HOT = {
    # prefill forward (fused window path)
    "omni::(anonymous namespace)::k_router_tc<256>": 0,
    "omni::(anonymous namespace)::k_select<32, 2, 2>": 0,
    "omni::(anonymous namespace)::k_prep<2>": 0,
    "omni::(anonymous namespace)::k_scan_reduce": 0,
    "omni::(anonymous namespace)::k_scan_tiles": 0,
    "omni::(anonymous namespace)::k_scan_finish": 0,
    "omni::(anonymous namespace)::k_wincount<2>": 0,
    "omni::(anonymous namespace)::k_rowscan": 0,
    "omni::(anonymous namespace)::k_winscatter<2>": 0,
    "omni::(anonymous namespace)::k_wsort_x": 0,
    "omni::(anonymous namespace)::k_act<__nv_bfloat16, 8, 3, ": 0,
    "omni::(anonymous namespace)::k_acc<__nv_bfloat16, 4, 4>": 0,
    "omni::(anonymous namespace)::k_slice_finish": 0,
    "omni::(anonymous namespace)::k_zero_words": 0,
    # decode forward
    "omni::(anonymous namespace)::k_router_tc<64>": 0,
    "omni::(anonymous namespace)::k_select_wide<8, 2, 2>": 16,
    "omni::(anonymous namespace)::k_task_act<__nv_bfloat16, 8, false>": 0,
    "omni::(anonymous namespace)::k_gather_v<__nv_bfloat16, 2, __nv_bfloat16>": 0,
    "omni::(anonymous namespace)::k_gather_v<__nv_bfloat16, 2, float>": 0,
    # decode stages timed separately (omni_schedule + omni_expert_forward)
    "omni::(anonymous namespace)::k_sched_bits<64>": 0,
    "omni::(anonymous namespace)::k_expert_async<__nv_bfloat16, 8, 3, false>": 0,
    "omni::(anonymous namespace)::k_cast": 0,
    # gated experts (SwiGLU) on the same paths
    "omni::(anonymous namespace)::k_task_act<__nv_bfloat16, 8, true>": 0,
    "omni::(anonymous namespace)::k_act<__nv_bfloat16, 8, 3, true, true>": 0,
    "omni::(anonymous namespace)::k_expert_async<__nv_bfloat16, 8, 2, true>": 0,
    # backward
    "omni::(anonymous namespace)::k_bwd_expert": 0,
    "omni::(anonymous namespace)::k_bwd_token": 0,
    "omni::(anonymous namespace)::k_transpose16": 0,
    # shards
    "omni::(anonymous namespace)::k_shard_range": 0,
}


def _parse(text):
    """{mangled entry name: {"regs", "spill"}} from one ptxas -v report."""
    out, entry, props = {}, None, None
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            entry = m.group(1)
            out[entry] = {"regs": None, "spill": None}
            continue
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            props = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and props in out:
            out[props]["spill"] = int(m.group(1)) + int(m.group(2))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry in out:
            out[entry]["regs"] = int(m.group(1))
    return out


@pytest.fixture(scope="module")
def kernels():
    libbuild.build()
    paths = [libbuild.report(s) for s in libbuild.sources()]
    if not all(os.path.exists(p) for p in paths):
        libbuild.build(force=True)  # objects built before the build kept reports
    found = {}
    for p in paths:
        with open(p) as fh:
            found.update(_parse(fh.read()))
    names = list(found)
    demangled = subprocess.run(["c++filt"], input="\n".join(names), capture_output=True,
                               text=True, check=True).stdout.splitlines()
    return {d.replace("void ", "", 1): found[n] for n, d in zip(names, demangled)}


def test_reports_cover_every_kernel(kernels):
    assert len(kernels) > 50
    assert all(k["regs"] is not None and k["spill"] is not None for k in kernels.values())


def test_benchmarked_kernels_do_not_spill(kernels):
    for prefix, allowed in HOT.items():
        hits = {n: k for n, k in kernels.items() if n.startswith(prefix)}
        assert hits, f"no kernel named {prefix}... (renamed?)"
        for n, k in hits.items():
            assert k["spill"] <= allowed, f"{n}: {k['spill']} bytes of spill"
            assert k["regs"] <= 255, n
