"""Expert-sharded forward across processes, one per GPU.

The N atomic experts are split into contiguous id ranges, one per process,
and each process holds only its range's rows of W and V (and U).  The
routing is replicated: every process routes the whole batch (the router
weights are small).  Each process then executes only the tasks of its own
experts, in the library's expert-centric order, and leaves an fp32 partial
output.  One all-reduce over the process group sums the partials, and a
cast rounds the sum to the storage type.

Compared with data-parallel replicas, this divides the expert rows that
each GPU must hold and stream by the group size.  The price is that the
route and the schedule are computed on every process, plus one all-reduce
of an L x d fp32 tensor.  The pages describe no distribution; this is the
split that the expert-centric order suggests.  Groups of B consecutive
active ids fall to the process that holds them, and a group on a range
boundary is executed by the processes on either side, each for its own ids.
"""
from __future__ import annotations

import contextlib

import torch

from . import LayerDims, cast_output, moe_forward_shard


def shard_ranges(N: int, G: int) -> list[tuple[int, int]]:
    """The contiguous split of ids [0, N) into G ranges whose sizes differ by
    at most one (the first N mod G ranges one larger)."""
    if G < 1 or N < G:
        raise ValueError(f"cannot split {N} ids into {G} non-empty ranges")
    q, r = divmod(N, G)
    out, lo = [], 0
    for g in range(G):
        hi = lo + q + (1 if g < r else 0)
        out.append((lo, hi))
        lo = hi
    return out


def combine(y_part: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the processes' partial outputs in place (one all-reduce of fp32)."""
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y_part, op=dist.ReduceOp.SUM, group=group)
    return y_part


def forward(D: LayerDims, x, Wr, Wc, W_shard, V_shard, e_lo: int, e_hi: int, bias_r=None,
            bias_c=None, *, U_shard=None, group=None, y=None, y_part=None, counts=None,
            idx=None, gate=None, ws=None, stream=None):
    """The whole layer's routed output on every process of `group`, from
    this process' expert rows [e_lo, e_hi).  The processes' ranges must
    partition [0, N) (shard_ranges), and every process must pass the same
    x, router weights and biases."""
    y_part = moe_forward_shard(D, x, Wr, Wc, W_shard, V_shard, e_lo, e_hi, bias_r, bias_c,
                               U=U_shard, y_part=y_part, counts=counts, idx=idx, gate=gate,
                               ws=ws, stream=stream)
    # the collective is ordered after the shard's kernels on their stream
    with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
        combine(y_part, group)
    return cast_output(D, y_part, y=y, stream=stream)
