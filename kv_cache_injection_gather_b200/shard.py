"""Partitions of an inject batch over GPUs (host logic only).

The path has no exchange step: requests are independent, and so are KV heads
(each head's store rows go only to that head's cache rows).  Two partitions:

* replicas / request shards: a rank injects its own requests into its own
  cache with its own copy of the store (data-parallel serving replicas);
* head shards: a rank holds KV heads [h0, h1) of every fact and of the cache
  (tensor-parallel serving shards its KV heads this way) and injects the
  whole batch for those heads.

Neither needs a collective on the data path.
"""
from __future__ import annotations

import numpy as np


def contiguous_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, end) of rank's share when n items are split as evenly as
    possible into world contiguous parts (the first n % world get one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def head_shard(num_kv_heads: int, world: int, rank: int) -> tuple[int, int]:
    if num_kv_heads % world:
        raise ValueError("KV heads must divide evenly over the ranks")
    return contiguous_range(num_kv_heads, world, rank)


def request_shard(req_offsets, fact_ids, start_pos, block_tables, world: int, rank: int):
    """The sub-batch of rank's contiguous run of requests (CSR re-based)."""
    R = len(start_pos)
    r0, r1 = contiguous_range(R, world, rank)
    ro = np.asarray(req_offsets, np.int64)
    ids = np.asarray(fact_ids)[ro[r0]:ro[r1]].astype(np.int32)
    sub_off = (ro[r0:r1 + 1] - ro[r0]).astype(np.int32)
    return (sub_off, ids, np.asarray(start_pos, np.int32)[r0:r1].copy(),
            np.asarray(block_tables, np.int32)[r0:r1].copy(), (r0, r1))
