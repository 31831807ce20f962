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

from . import LayerDims, cast_output, moe_forward_shard, moe_forward_shard_routed, route


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


def token_ranges(L: int, G: int) -> list[tuple[int, int]]:
    """Process g routes tokens [g*T, min((g+1)*T, L)), T = ceil(L / G)
    (the last ranges may be short or empty)."""
    if G < 1:
        raise ValueError("a group has at least one process")
    T = -(-L // G)
    return [(min(g * T, L), min((g + 1) * T, L)) for g in range(G)]


def gather_routing(idx_part: torch.Tensor, gate_part: torch.Tensor, L: int, group=None):
    """The whole batch's routing from every process's share (token_ranges):
    one all-gather of the ids and one of the gates, each share padded to
    ceil(L / G) rows.  Returns (idx [L, K], gate [L, K])."""
    import torch.distributed as dist
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    if G == 1:
        return idx_part, gate_part
    K = idx_part.shape[1]
    T = -(-L // G)
    outs = []
    for part in (idx_part, gate_part):
        padded = torch.zeros((T, K), dtype=part.dtype, device=part.device)
        padded[: part.shape[0]] = part
        full = torch.empty((G * T, K), dtype=part.dtype, device=part.device)
        dist.all_gather_into_tensor(full, padded, group=group)
        outs.append(full[:L].contiguous())
    return outs[0], outs[1]


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


def forward_split_routing(D: LayerDims, x, Wr, Wc, W_shard, V_shard, e_lo: int, e_hi: int,
                          bias_r=None, bias_c=None, *, U_shard=None, group=None, y=None,
                          y_part=None, counts=None, ws=None, stream=None):
    """forward() with the routing split as well: process g routes only its
    tokens (token_ranges), the shares are all-gathered, and each process
    then schedules and executes its experts from the whole routing.  The
    route is computed once per token in the group instead of once per
    process."""
    import torch.distributed as dist
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    g = dist.get_rank(group) if dist.is_initialized() else 0
    t0, t1 = token_ranges(D.L, G)[g]
    Dg = LayerDims(t1 - t0, D.d, D.Nr, D.Nc, D.k, D.K, D.B, D.dtype, D.flags)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    if t1 > t0:
        idx_part, gate_part, _ = route(Dg, x[t0:t1], Wr, Wc, bias_r, bias_c, with_score=False,
                                       stream=stream)
    else:
        idx_part = torch.empty((0, D.K), dtype=torch.int32, device=x.device)
        gate_part = torch.empty((0, D.K), dtype=torch.float32, device=x.device)
    with ctx:
        idx, gate = gather_routing(idx_part, gate_part, D.L, group)
    y_part = moe_forward_shard_routed(D, x, W_shard, V_shard, e_lo, e_hi, idx, gate,
                                      U=U_shard, y_part=y_part, counts=counts, ws=ws,
                                      stream=stream)
    with ctx:
        combine(y_part, group)
    return cast_output(D, y_part, y=y, stream=stream)
