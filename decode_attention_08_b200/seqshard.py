"""One long sequence's cache split across GPUs (sequence parallelism at decode).

Each rank holds a contiguous key range of every sequence and attends over it
with ``mfa.decode_attention_ex`` (f32 output and log-sum-exp); the (O, lse)
parts of all ranks are all-gathered and merged by ``mfa.lse_merge``
(Flash-Decoding's combine, cited on the DeepSeek-V4 page's reference list). The
one exchange is B x 64 x 257 floats per rank (the normalised output and the lse
of each head), against the rank's B x L/N x 1 KB of cache read.

This module is host-side plumbing only: every arithmetic step runs in
``libmfa.so``; torch.distributed (NCCL on GPUs, gloo in the CPU tests) moves the
parts.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import mfa

TILE = 128  # tokens per attention tile: ranges are cut at tile boundaries


def key_range(length: int, rank: int, world: int, align: int = TILE) -> Tuple[int, int]:
    """Token range [start, stop) of ``rank`` when a sequence of ``length`` cached
    tokens is split over ``world`` ranks: contiguous, disjoint, covering, cut at
    multiples of ``align`` tokens, the tiles spread as evenly as possible (the
    first ``tiles % world`` ranks take one more); ranks past the end get an
    empty range at ``length``."""
    if world < 1 or not 0 <= rank < world or length < 0 or align < 1:
        raise ValueError("key_range: bad arguments")
    tiles = -(-length // align)
    base, extra = divmod(tiles, world)
    first = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return min(first * align, length), min((first + count) * align, length)


def local_lengths(seq_lens, rank: int, world: int, align: int = TILE):
    """Per-sequence (start, count) of this rank's key range: two int lists."""
    starts, counts = [], []
    for L in (int(x) for x in seq_lens):
        a, e = key_range(L, rank, world, align)
        starts.append(a)
        counts.append(e - a)
    return starts, counts


def gather_parts(o_part: torch.Tensor, lse_part: torch.Tensor, group=None):
    """All-gather every rank's (O [B, 64, 256] f32, lse [B, 64] f32) part, in
    rank order: returns (o_parts [S, B, 64, 256], lse_parts [S, B, 64])."""
    world = dist.get_world_size(group)
    o_parts = o_part.new_empty((world,) + tuple(o_part.shape))
    lse_parts = lse_part.new_empty((world,) + tuple(lse_part.shape))
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(o_parts, o_part.contiguous(), group=group)
        dist.all_gather_into_tensor(lse_parts, lse_part.contiguous(), group=group)
    else:
        dist.all_gather(list(o_parts.unbind(0)), o_part.contiguous(), group=group)
        dist.all_gather(list(lse_parts.unbind(0)), lse_part.contiguous(), group=group)
    return o_parts, lse_parts


def sharded_decode(q, k_local, v_local, local_lens, out, *, group=None,
                   softmax_scale: float = 1.0 / 16, kv_dtype: str = "bf16",
                   k_scale: float = 1.0, v_scale: float = 1.0, page_table=None,
                   lse_out: Optional[torch.Tensor] = None, workspace=None):
    """Decode attention of sequences whose caches are split across the ranks of
    ``group``: this rank's cache ``k_local``/``v_local`` holds ``local_lens[b]``
    tokens of sequence b (its range from ``key_range``); q is the same on every
    rank. Every rank ends with the full result in ``out`` (and ``lse_out``).
    Everything runs on the current stream, the one the collectives use."""
    B = q.shape[0]
    o_part = torch.empty(B, q.shape[1], q.shape[2], dtype=torch.float32, device=q.device)
    lse_part = torch.empty(B, q.shape[1], dtype=torch.float32, device=q.device)
    mfa.decode_attention_ex(q, k_local, v_local, page_table, local_lens, o_part, softmax_scale,
                            kv_dtype, k_scale, v_scale, 0, lse_part, workspace)
    o_parts, lse_parts = gather_parts(o_part, lse_part, group)
    return mfa.lse_merge(o_parts, lse_parts, out, lse_out)
