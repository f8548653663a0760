"""Decode spread over several GPUs: one process per GPU under torch.distributed.

Two ways to spread one decode step, both from "现代 LLM 的 Memory-Compute
Trade-off：从 MHA 到 MLA" (section "MHA 与 KV Cache": the cache grows linearly
with the sequence, so long contexts outgrow one device) and "Transformer升级之路：
21、MLA好在哪里?（下）" (section 总而言之: MQA-form decoding cannot be split by
head, since every head reads the same latent cache):

* batch sharding: each rank decodes its own contiguous slice of the sequences
  with mla_decode; nothing is exchanged.
* key-range sharding (split-KV across devices) for one long sequence: each rank
  holds the pages of one key range, computes its partial with
  mla_decode_partial, the partials (o_lat and lse, a few KB per query token)
  are all-gathered, and every rank merges them exactly with mla_merge_partials.

The collective is the only cross-device step; the arithmetic runs in libmla.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def batch_shard(batch: int, world: int, rank: int) -> tuple:
    """The [start, stop) slice of sequences rank `rank` decodes: contiguous, sizes differ by at most one."""
    if not (0 <= rank < world) or batch < 0:
        raise ValueError("bad rank, world or batch")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def kv_shard_ranges(max_seqlen: int, world: int, align: int = 64) -> list:
    """Key ranges [begin, end) of the ranks: they cover 0 .. max_seqlen, begins are multiples of
    `align` (the attention kernel reads whole 64-token pages), and their sizes differ by at most
    one page.  A rank may get an empty range when there are fewer pages than ranks."""
    if world <= 0 or max_seqlen <= 0 or align <= 0:
        raise ValueError("bad world, max_seqlen or align")
    pages = (max_seqlen + align - 1) // align
    out = []
    for r in range(world):
        p0, p1 = r * pages // world, (r + 1) * pages // world
        out.append((p0 * align, min(p1 * align, max_seqlen) if p1 > p0 else p0 * align))
    return out


def gather_partials(o_lat: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's partial: returns ([world, *o_lat.shape], [world, *lse.shape]) in rank order."""
    world = dist.get_world_size(group)
    # Gathered along dim 0 (the form every backend accepts), then viewed as [world, ...].
    o_all = o_lat.new_empty((world * o_lat.shape[0],) + tuple(o_lat.shape[1:]))
    l_all = lse.new_empty((world * lse.shape[0],) + tuple(lse.shape[1:]))
    dist.all_gather_into_tensor(o_all, o_lat.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse.contiguous(), group=group)
    return o_all.view((world,) + tuple(o_lat.shape)), l_all.view((world,) + tuple(lse.shape))


def split_kv_decode(mla, dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                    max_seqlen, w_uk, w_uv, out, lse=None, group=None, dev_status=None):
    """One decode step whose keys are split over the ranks of `group` by kv_shard_ranges.

    Every rank passes the same queries, seqlens and weights, and a block table whose entries for
    the pages of its own key range point into its local pool (entries outside the range are never
    read).  Every rank ends with the full result in `out` (and `lse`)."""
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    kv_begin, kv_end = kv_shard_ranges(max_seqlen, world)[rank]
    B, n_q, H = q_nope.shape[:3]
    o_lat = torch.empty((B, n_q, H, dims.d_c), dtype=q_nope.dtype, device=q_nope.device)
    part_lse = torch.empty((B, n_q, H), dtype=torch.float32, device=q_nope.device)
    if kv_end > kv_begin:
        ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
        mla.mla_decode_partial(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                               max_seqlen, kv_begin, kv_end, w_uk, o_lat, part_lse, ws, dev_status)
    else:                                     # no keys on this rank: a neutral partial
        o_lat.zero_()
        part_lse.fill_(float("-inf"))
    o_all, l_all = gather_partials(o_lat, part_lse, group)
    mws = mla.alloc_workspace(mla.mla_merge_workspace_size(dims, B, n_q, world))
    mla.mla_merge_partials(dims, o_all, l_all, w_uv, out, lse, mws)
