"""One prefill chunk split by queries over several GPUs (one process per GPU).

Query rows are independent given the cache, so rank r runs dsa_prefill_layer
on its own contiguous query range (cut by dsa_partition_queries so that every
rank gets nearly the same useful work) against the whole cache. Two exchanges
surround the layer, both plain torch.distributed collectives (NCCL over
NVLink on GPUs, gloo on CPU):

  1. the chunk's new cache rows: each rank produced the latent, rope and
     indexer-key rows of its own queries (cache rows q_pos0 + start ..
     q_pos0 + end - 1), and every rank needs all of them before its layer;
  2. the outputs: each rank's out rows (and lse, idx when asked) gathered
     into the full chunk, for a consumer that is not itself split by queries.

Ranges differ in length, so each collective moves row blocks padded to the
longest range and drops the padding on arrival. This module holds no part of
the layer's arithmetic; the layer itself is the caller's function (the CUDA
library on GPUs).
"""
from __future__ import annotations

import dataclasses

from . import check, dsa_partition_queries


def query_ranges(dims, world: int) -> list[tuple[int, int]]:
    """(start, end) query rows of every rank, from dsa_partition_queries."""
    st, starts = dsa_partition_queries(dims, world)
    check(st)
    return [(starts[r], starts[r + 1]) for r in range(world)]


def sub_dims(dims, start: int, end: int):
    """The dims of rows start .. end-1 of a chunk (same cache, shifted q_pos0)."""
    return dataclasses.replace(dims, n_q=end - start, q_pos0=dims.q_pos0 + start)


def gather_row_blocks(full, ranges, rank: int, row0: int = 0, group=None):
    """All-gather of contiguous row blocks of `full` (in place).

    Rank r owns rows row0 + start_r .. row0 + end_r - 1 of `full` (its own
    block is already in place); afterwards every rank holds every block. The
    blocks are padded to the longest range for the collective."""
    import torch
    import torch.distributed as dist

    world = len(ranges)
    longest = max(e - s for s, e in ranges)
    if world == 1 or longest == 0:
        return full
    s, e = ranges[rank]
    row_shape = full.shape[1:]
    send = torch.zeros((longest, *row_shape), dtype=full.dtype, device=full.device)
    send[: e - s] = full[row0 + s: row0 + e]
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    for r, (rs, re_) in enumerate(ranges):
        if r != rank and re_ > rs:
            full[row0 + rs: row0 + re_] = recv[r][: re_ - rs]
    return full


def prefill_layer_sharded(dims, rank: int, world: int, cache: dict, chunk: dict, outputs: dict,
                          layer_fn, gather_outputs: bool = True, group=None):
    """One query-split step of the layer on this rank.

    cache:   {"latent", "rope", "k_idx"} full-context tensors [ctx_len, ...];
             this rank's own chunk rows are already written, the other
             ranks' chunk rows arrive through the first exchange.
    chunk:   {"q", "q_idx", "w_idx"} full-chunk tensors [n_q, ...]; only this
             rank's rows are read.
    outputs: {"out", optionally "lse", "idx"} full-chunk tensors [n_q, ...];
             this rank's rows are written by layer_fn, the others arrive
             through the second exchange (when gather_outputs).
    layer_fn(sub_dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx)
             runs the layer on one query range (row slices of the chunk and
             output tensors, the whole cache).
    Returns this rank's (start, end)."""
    ranges = query_ranges(dims, world)
    s, e = ranges[rank]
    for key in ("latent", "rope", "k_idx"):
        gather_row_blocks(cache[key], ranges, rank, row0=dims.q_pos0, group=group)
    if e > s:
        layer_fn(sub_dims(dims, s, e), chunk["q"][s:e], cache["latent"], cache["rope"],
                 chunk["q_idx"][s:e], cache["k_idx"], chunk["w_idx"][s:e],
                 outputs["out"][s:e],
                 outputs["lse"][s:e] if outputs.get("lse") is not None else None,
                 outputs["idx"][s:e] if outputs.get("idx") is not None else None)
    if gather_outputs:
        for key in ("out", "lse", "idx"):
            if outputs.get(key) is not None:
                gather_row_blocks(outputs[key], ranges, rank, group=group)
    return s, e
