"""Context parallelism for decode: each rank holds a contiguous stretch of
every sequence's keys and values, attends over it with the local plan, and
one all-gather of the (out, lse) pairs followed by a local log-sum-exp merge
(`merge_lse`, the C ABI's attn_merge_lse) gives every rank the full result.
This is the exchange step of a sequence split over GPUs: the partial states
of the kernbench2 docs/adr-proposed commit log (GQA entry: running
(m, l, O) reduced between devices), carried as normalised (out, lse) pairs so
that the local kernels need no change, with one collective instead of the
page's log-N tree of sends (on NVSwitch a single all-gather of these few
kilobytes costs one collective's latency, a tree costs log N of them).

Decode only (q_len = 1 in every sequence): the tail-aligned causal mask is
then a no-op, so keys may be split anywhere.  The product path runs the local
attention and the merge in libvgqa's kernels; `attend` and `merge` can be
replaced, which the CPU tests use to drive the exchange logic over gloo.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from ._binding import merge_lse


def shard_bounds(cu_k: torch.Tensor, rank: int, world: int):
    """Per sequence, the rank's key range [lo, hi) in packed token indexes:
    rank r holds keys [floor(Lk r / world), floor(Lk (r + 1) / world)) of a
    sequence with Lk keys, so the ranks' ranges tile it in order."""
    cu = cu_k.to(torch.int64)
    lens = cu[1:] - cu[:-1]
    lo = cu[:-1] + (lens * rank) // world
    hi = cu[:-1] + (lens * (rank + 1)) // world
    return lo, hi


def shard_kv(k: torch.Tensor, v: torch.Tensor, cu_k: torch.Tensor, rank: int, world: int):
    """This rank's keys and values, packed, with their cu_seqlens.  Setup-time
    (it reads the lengths on the host), not part of a decode step."""
    lo, hi = shard_bounds(cu_k, rank, world)
    lo_h, hi_h = lo.cpu().tolist(), hi.cpu().tolist()
    idx = torch.cat([torch.arange(a, b, dtype=torch.int64) for a, b in zip(lo_h, hi_h)] +
                    [torch.zeros(0, dtype=torch.int64)]).to(k.device)
    lens = torch.tensor([b - a for a, b in zip(lo_h, hi_h)], dtype=torch.int64)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    k_loc = k.index_select(0, idx).contiguous()
    v_loc = v.index_select(0, idx).contiguous()
    return k_loc, v_loc, cu.to(cu_k.device)


def _all_gather(x: torch.Tensor, world: int, group) -> torch.Tensor:
    out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    try:
        dist.all_gather_into_tensor(out.view((world * x.shape[0],) + tuple(x.shape[1:])), x, group=group)
    except (RuntimeError, NotImplementedError, ValueError):
        dist.all_gather(list(out.unbind(0)), x, group=group)
    return out


def decode_step(plan, q, k_loc, v_loc, cu_q, cu_k_loc, *, group=None, out=None, lse=None, attend=None,
                merge=None):
    """One context-parallel decode step on this rank: local attention over its
    key shard, all-gather of (out, lse) across the group (rank order), merge.
    Returns the merged (out, lse), the same on every rank."""
    world = dist.get_world_size(group)
    if attend is None:
        o_loc, l_loc = plan.run(q, k_loc, v_loc, cu_q, cu_k_loc)
    else:
        o_loc, l_loc = attend(q, k_loc, v_loc, cu_q, cu_k_loc)
    outs = _all_gather(o_loc.contiguous(), world, group)
    lses = _all_gather(l_loc.contiguous(), world, group)
    if merge is None:
        return merge_lse(outs, lses, cu_q, out=out, lse=lse)
    return merge(outs, lses, cu_q)
