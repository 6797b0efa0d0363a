"""Decode context parallelism (DCP) over N ranks, host side.

The beaiera.top DeepSeek tag page (the abstract on DCP and on MLA prefill vs
decode) describes sharding the KV cache of each sequence along the sequence
across ranks. Here each rank holds contiguous runs of whole 64-token pages of
every sequence; rank r decodes its run with the library (``mla_decode_plan``
/ ``mla_decode`` / ``mla_combine``), the ranks' ``(out, lse)`` are
all-gathered, and ``mla_merge`` combines them by LSE. The merge is exact in
the sense of the split-KV combine: ``lse = ln sum_r exp(lse_r)``,
``out = sum_r exp(lse_r - lse) out_r``.

Sharding rule (``shard_bounds``): sequence b has P = ceil(L_b / 64) pages.
The last rank holds the tail, [s_last, P) with s_last = P - ceil(P / N),
moved earlier when needed so that it holds every token some causal query
cannot see (the last Sq - 1 tokens); the first N - 1 ranks split [0, s_last)
into near-equal contiguous runs. A rank's tokens are renumbered from 0 and
its block-table row lists its pages, so a causal step runs causal only on
the last rank (every token before the tail is visible to every query row),
and a sparse step maps each listed position into the owning rank's run (-1
elsewhere).

``decode`` and ``merge`` default to the library on the rank's GPU; the
gather uses ``torch.distributed`` (NCCL between GPUs). Nothing here does
attention arithmetic.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch

PAGE = 64


def shard_bounds(seq_len: int, world: int, *, q_len: int = 1, causal: bool = False):
    """Page runs ``[(p0, p1)]`` of one sequence for ranks 0..world-1."""
    P = (max(int(seq_len), 0) + PAGE - 1) // PAGE
    chunk = (P + world - 1) // world
    s_last = max(P - chunk, 0)
    if causal and q_len > 1 and seq_len >= q_len:
        s_last = min(s_last, (seq_len - q_len) // PAGE)  # the last Sq - 1 tokens sit on the last rank
    runs = []
    head = world - 1
    for r in range(head):
        runs.append((s_last * r // head, s_last * (r + 1) // head))
    runs.append((s_last, P))
    return runs


def shard_inputs(block_table: torch.Tensor, seq_lens: torch.Tensor, *, world: int, rank: int, q_len: int = 1,
                 causal: bool = False, indices: Optional[torch.Tensor] = None) -> dict:
    """The block table, lengths, causal flag and (sparse) positions of rank
    ``rank``'s shard. ``block_table [B, maxp]`` page ids, ``seq_lens [B]``,
    ``indices [B, Sq, topk]`` logical positions or None. Tensors stay on
    their device; the computation is index bookkeeping only."""
    dev = block_table.device
    lens = [int(x) for x in seq_lens.tolist()]
    B = len(lens)
    runs = [shard_bounds(L, world, q_len=q_len, causal=causal)[rank] for L in lens]
    maxp = max([p1 - p0 for p0, p1 in runs] + [1])
    bt = torch.zeros(B, maxp, dtype=torch.int32, device=dev)
    local_lens = torch.zeros(B, dtype=torch.int32)
    starts = torch.zeros(B, dtype=torch.int64)
    ends = torch.zeros(B, dtype=torch.int64)
    for b, (p0, p1) in enumerate(runs):
        if p1 > p0:
            bt[b, :p1 - p0] = block_table[b, p0:p1]
        starts[b] = p0 * PAGE
        ends[b] = min(lens[b], p1 * PAGE)
        local_lens[b] = max(int(ends[b] - starts[b]), 0)
    local_idx = None
    if indices is not None:
        idx = indices.to(torch.int64)
        lo = starts.to(idx.device)[:, None, None]
        hi = ends.to(idx.device)[:, None, None]
        inside = (idx >= lo) & (idx < hi)
        local_idx = torch.where(inside, idx - lo, torch.full_like(idx, -1)).to(torch.int32)
    return {"block_table": bt, "seq_lens": local_lens.to(dev), "indices": local_idx,
            "causal": bool(causal) and rank == world - 1, "starts": starts, "max_pages_per_seq": maxp}


def _library_decode(q, kv_cache, shard):
    from .decoder import MlaDecoder

    B, Sq, H, _ = q.shape
    dec = MlaDecoder(batch=B, q_len=Sq, num_heads=H, num_pages=kv_cache.shape[0],
                     max_pages_per_seq=shard["max_pages_per_seq"],
                     topk=0 if shard["indices"] is None else shard["indices"].shape[-1], causal=shard["causal"],
                     device=q.device)
    out, lse = dec(q, kv_cache, shard["block_table"], shard["seq_lens"], shard["indices"])
    return out.clone(), lse.clone()


def library_merge(part_out: torch.Tensor, part_lse: torch.Tensor):
    """``mla_merge`` of ``part_out [N, ..., 512]`` bf16 and ``part_lse [N, ...]`` on their GPU."""
    from . import binding as Bd

    N = part_out.shape[0]
    rows = part_lse[0].numel()
    out = torch.empty(part_out.shape[1:], dtype=torch.bfloat16, device=part_out.device)
    lse = torch.empty(part_lse.shape[1:], dtype=torch.float32, device=part_out.device)
    with torch.cuda.device(part_out.device):
        Bd.check(Bd.mla_merge(Bd.make_merge_desc(parts=N, rows=rows), part_out.contiguous(), part_lse.contiguous(),
                              out, lse, torch.cuda.current_stream(part_out.device)), "mla_merge")
    return out, lse


def dcp_decode(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor, *,
               world: int, rank: int, q_len: int = 1, causal: bool = False,
               indices: Optional[torch.Tensor] = None, group=None,
               decode: Optional[Callable] = None, merge: Optional[Callable] = None):
    """One decode step of rank ``rank`` of ``world`` under DCP: decode this
    rank's shard, all-gather every rank's ``(out, lse)`` and merge them.
    Every rank calls it with the same arguments (the full block table and
    lengths; a rank reads only its own pages of ``kv_cache``). Returns the
    merged ``(out, lse)`` on every rank. A rank that left the group makes the
    gather raise here (after the process group's timeout at the latest)."""
    import torch.distributed as dist

    shard = shard_inputs(block_table, seq_lens, world=world, rank=rank, q_len=q_len, causal=causal, indices=indices)
    out_r, lse_r = (decode or _library_decode)(q, kv_cache, shard)
    if world > 1:
        outs = [torch.empty_like(out_r) for _ in range(world)]
        lses = [torch.empty_like(lse_r) for _ in range(world)]
        dist.all_gather(outs, out_r.contiguous(), group=group)
        dist.all_gather(lses, lse_r.contiguous(), group=group)
    else:
        outs, lses = [out_r], [lse_r]
    return (merge or library_merge)(torch.stack(outs), torch.stack(lses))
