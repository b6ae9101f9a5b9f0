"""Split-KV decode across ranks (one process per GPU, torch.distributed).

Each of R ranks holds a contiguous part of every request's KV pages in its own
pool and decodes the same queries against it with the single-GPU path; the
ranks then exchange their results (fp32 O before any bf16 rounding, and fp32
LSE; one all-gather each, over NVLink with NCCL) and every rank merges them
with ``mla_decode_combine_ranks_f32``: L* = log sum_i exp(lse_i), O = sum_i
exp(lse_i - L*) O_i, rounded to bf16 once, as the combine of split partials
inside one GPU does.  That exchange is the one collective the path needs when
a single request's context is spread over several GPUs; batches that fit one
GPU shard over requests instead, with no collective at all.

Page split: request b with P_b pages gives rank r the pages
[floor(r P_b / R), floor((r + 1) P_b / R)), so the last rank always holds the
request's last page.  The causal rule with s_q new tokens hides the request's
last s_q - 1 positions from its earlier query tokens.  With s_q <= 2 that is
at most the last position, which lies in the last page, so only the last rank
applies the causal rule and every other rank's tokens are visible to all query
tokens.  (With s_q >= 3 the hidden positions could straddle a rank boundary;
the decode library takes s_q 1 or 2 only, and so does this split.)
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import binding as bd

PAGE_SIZE = bd.PAGE_SIZE


def page_range(num_pages: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous page range [p0, p1) of ``rank`` for a request of ``num_pages``."""
    if world < 1 or not 0 <= rank < world or num_pages < 0:
        raise ValueError("bad split: pages %d, world %d, rank %d" % (num_pages, world, rank))
    return (rank * num_pages) // world, ((rank + 1) * num_pages) // world


def check_s_q(s_q: int) -> None:
    """The split's causal assignment holds for one or two new tokens only."""
    if s_q not in (1, 2):
        raise ValueError("split-KV across ranks takes s_q 1 or 2, got %r" % (s_q,))


def rank_causal(causal: bool, world: int, rank: int) -> bool:
    """Whether ``rank`` applies the causal rule: only the holder of the tails
    (exact for s_q <= 2, see the module docstring)."""
    return bool(causal) and rank == world - 1


def shard(cache_seqlens: torch.Tensor, block_table: torch.Tensor, world: int,
          rank: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's part of a paged batch: (local cache_seqlens int32 [B],
    local block_table int32 [B, max local pages], -1 past each request's
    pages).  Host tensors in, host tensors out; the page ids are those of the
    global table (a rank that keeps its own pool renumbers them)."""
    sl = cache_seqlens.to("cpu", torch.int64)
    bt = block_table.to("cpu", torch.int32)
    B = sl.shape[0]
    ranges = []
    for b in range(B):
        L = max(int(sl[b]), 0)
        P = (L + PAGE_SIZE - 1) // PAGE_SIZE
        ranges.append((L, page_range(P, world, rank)))
    width = max([p1 - p0 for _, (p0, p1) in ranges] + [1])
    local_bt = torch.full((B, width), -1, dtype=torch.int32)
    local_sl = torch.zeros(B, dtype=torch.int32)
    for b, (L, (p0, p1)) in enumerate(ranges):
        local_bt[b, :p1 - p0] = bt[b, p0:p1]
        local_sl[b] = max(0, min(PAGE_SIZE * p1, L) - PAGE_SIZE * p0)
    return local_sl, local_bt


def gather(local: torch.Tensor, group=None) -> torch.Tensor:
    """Stack of every rank's ``local`` (same shape everywhere), rank-major."""
    world = dist.get_world_size(group)
    full = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(full, local.contiguous(), group=group)
    else:  # gloo (CPU tests) gathers into a list of views
        dist.all_gather(list(full.unbind(0)), local.contiguous(), group=group)
    return full


class KvSplitDecoder:
    """One rank's part of an MLA decode whose KV is split across the ranks of
    ``group``: local decode (fp32 output), all-gather of (O, LSE), merge.  Shapes as for
    ``MlaDecoder``; ``num_blocks`` / ``max_blocks_per_seq`` describe this
    rank's pool and local block table."""

    def __init__(self, batch: int, s_q: int, num_heads: int, num_blocks: int, max_blocks_per_seq: int,
                 causal: bool = False, group=None, device: Optional[torch.device] = None):
        check_s_q(s_q)
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.dec = bd.MlaDecoder(batch, s_q, num_heads, num_blocks, max_blocks_per_seq,
                                 rank_causal(causal, self.world, self.rank), device=device, fp32_out=True)
        dev = self.dec.device
        self.out = torch.empty(batch, s_q, num_heads, bd.D_V, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(batch, num_heads, s_q, dtype=torch.float32, device=dev)

    def plan(self, local_seqlens: torch.Tensor) -> None:
        self.dec.plan(local_seqlens)

    def __call__(self, q, kv_local, block_table_local, seqlens_local,
                 softmax_scale: float) -> Tuple[torch.Tensor, torch.Tensor]:
        o, l = self.dec(q, kv_local, block_table_local, seqlens_local, softmax_scale)
        o_all = gather(o, self.group)
        l_all = gather(l, self.group)
        bd.mla_decode_combine_ranks(o_all, l_all, self.out, self.lse)
        return self.out, self.lse


class KvSplitGqaDecoder:
    """The same split for the GQA path over a group-expanded cache: every
    rank holds a contiguous part of each request's pages (all KV groups of a
    token live in one row), decodes it with ``GqaDecoder``, and the ranks
    merge their 128-wide outputs by LSE."""

    def __init__(self, batch: int, s_q: int, num_kv_groups: int, num_blocks: int, max_blocks_per_seq: int,
                 causal: bool = False, group=None, device: Optional[torch.device] = None):
        check_s_q(s_q)
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.dec = bd.GqaDecoder(batch, s_q, num_kv_groups, num_blocks, max_blocks_per_seq,
                                 rank_causal(causal, self.world, self.rank), device=device, fp32_out=True)
        dev = self.dec.device
        h = self.dec.dims.num_q_heads
        self.out = torch.empty(batch, s_q, h, bd.GQA_D_HEAD, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(batch, h, s_q, dtype=torch.float32, device=dev)

    def plan(self, local_seqlens: torch.Tensor) -> None:
        self.dec.plan(local_seqlens)

    def __call__(self, q, kv_local, block_table_local, seqlens_local,
                 softmax_scale: float) -> Tuple[torch.Tensor, torch.Tensor]:
        o, l = self.dec(q, kv_local, block_table_local, seqlens_local, softmax_scale)
        bd.mla_decode_combine_ranks(gather(o, self.group), gather(l, self.group), self.out, self.lse)
        return self.out, self.lse
