"""Partitions of an inject batch over the GPUs of a node (host logic).

Requests are independent, and so are KV heads (each head's store rows go
only to that head's cache rows).  Three partitions:

* replicas / request shards: a rank injects its own requests into its own
  cache with its own copy of the store (data-parallel serving replicas);
* head shards: a rank holds KV heads [h0, h1) of every fact and of the cache
  (tensor-parallel serving shards its KV heads this way) and injects the
  whole batch for those heads;
* fact shards: a rank holds a share of the facts (all layers and heads) and
  injects its own requests, whose facts live on every rank.  This is the one
  partition with an exchange: the inject kernel reads each remote fact's
  rows straight from the owner's arena over NVLink (peer loads through a
  CUDA IPC mapping), so the rows cross the link once and land in the cache
  with no staging copy.  FactShardGroup sets the view up.

The first two need no collective on the data path; the third needs none
either, only peer mappings made once at set-up.
"""
from __future__ import annotations

from typing import Callable, Sequence

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


def round_robin_owner(num_facts: int, world: int) -> np.ndarray:
    """Owner rank of every global fact id: g % world.  A rank puts its facts
    in increasing global id order, so g is local fact g // world there."""
    if world < 1 or num_facts < 0:
        raise ValueError("bad world/num_facts")
    return (np.arange(num_facts, dtype=np.int64) % world).astype(np.int32)


def owned_facts(owner: Sequence[int], rank: int) -> np.ndarray:
    """Global ids rank owns, in the order it puts them (increasing)."""
    return np.flatnonzero(np.asarray(owner) == rank).astype(np.int64)


def global_fact_table(owner: Sequence[int], local_tables: Sequence[tuple[Sequence[int], Sequence[int]]]):
    """The view's global fact table.

    owner[g] is the rank holding global fact g; local_tables[p] = (offsets,
    lengths) of rank p's local facts in its put order, which is increasing
    global id.  Returns (fact_shard int32, fact_offset int64, fact_len int32)
    over all global ids, the shard of a fact being its owner's rank."""
    owner = np.asarray(owner, dtype=np.int64)
    world = len(local_tables)
    if owner.size and (owner.min() < 0 or owner.max() >= world):
        raise ValueError("owner rank outside the group")
    shard = owner.astype(np.int32)
    off = np.zeros(owner.size, np.int64)
    ln = np.zeros(owner.size, np.int32)
    for p in range(world):
        ids = np.flatnonzero(owner == p)
        o = np.asarray(local_tables[p][0], np.int64)
        n = np.asarray(local_tables[p][1], np.int64)
        if len(o) != ids.size or len(n) != ids.size:
            raise ValueError(f"rank {p} holds {len(o)} facts, the owner map gives it {ids.size}")
        off[ids] = o
        ln[ids] = n
    return shard, off, ln


class FactShardGroup:
    """Attaches a fact-sharded view to this rank's store.

    Every rank of `group` calls this with its own store (device tier, its
    facts put in increasing global id order) and the same owner map.  The
    ranks swap their fact tables and their arenas' IPC handles (one
    all_gather_object on the host); each rank maps the peers' arenas into its
    process (is_ipc_open: peer access over NVLink) and attaches the view, so
    its batches take global fact ids.  close() is collective too: every rank
    must have finished its batches that read the view."""

    def __init__(self, store, owner: Sequence[int], group=None,
                 ipc_open: Callable[[int, bytes], int] | None = None,
                 ipc_close: Callable[[int, int], None] | None = None):
        import torch.distributed as dist
        if ipc_open is None or ipc_close is None:
            from . import binding as B
            ipc_open, ipc_close = ipc_open or B.is_ipc_open, ipc_close or B.is_ipc_close
        self._dist, self._group = dist, group
        self._open, self._close = ipc_open, ipc_close
        self.store = store
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        owner = np.asarray(owner, np.int32)
        n_local = store.num_facts
        if n_local != int((owner == self.rank).sum()):
            raise ValueError(f"rank {self.rank} holds {n_local} facts, the owner map gives it "
                             f"{int((owner == self.rank).sum())}")
        info = [store.fact_info(i) for i in range(n_local)]
        hk, hv, plane = store.export()
        mine = {"offsets": [o for o, _ in info], "lengths": [n for _, n in info],
                "k": hk, "v": hv, "plane": plane}
        everyone: list = [None] * self.world
        dist.all_gather_object(everyone, mine, group=group)
        self.opened: list[int] = []
        arenas = []
        try:
            for p, e in enumerate(everyone):
                if p == self.rank:
                    kp, vp, t = store.arena_ptrs()
                    arenas.append((kp, vp, t))
                else:
                    kp = self._open(store.device, e["k"])
                    self.opened.append(kp)
                    vp = self._open(store.device, e["v"])
                    self.opened.append(vp)
                    arenas.append((kp, vp, e["plane"]))
            table = global_fact_table(owner, [(e["offsets"], e["lengths"]) for e in everyone])
            store.attach_shards(arenas, *table)
        except Exception:
            self._unmap()
            raise
        self.arenas = arenas
        self.num_global_facts = int(owner.size)

    def _unmap(self) -> None:
        for ptr in self.opened:
            self._close(self.store.device, ptr)
        self.opened = []

    def close(self) -> None:
        """Collective: detach, unmap the peers' arenas, then wait for every
        rank to have unmapped ours (after which the stores may be freed)."""
        self._dist.barrier(group=self._group)
        self.store.detach_shards()
        self._unmap()
        self._dist.barrier(group=self._group)
