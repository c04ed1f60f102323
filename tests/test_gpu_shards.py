"""Fact-sharded stores on the GPU, through the C-ABI, against the CPU oracle.

A view over several stores' arenas (is_store_attach_shards) must inject
exactly what one store holding every fact injects: the oracle's result on
the full store, same bar as the other parity tests.  Here the shards are
stores on one GPU (local arena addresses), and in the two-process test
stores of two processes on one GPU, each mapping the other's arenas through
CUDA IPC (is_store_export / is_ipc_open) — the same kernel path peer GPUs
take over NVLink, where the mapped address is a peer's memory.
"""
from __future__ import annotations

import os
import socket
import sys
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from synth.device import make_store
from kv_cache_injection_gather_b200 import binding as B
from kv_cache_injection_gather_b200 import shard
from test_gpu_parity import PATHS, _need_gpu, _ragged, assert_parity, gpu_run, oracle_run

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _local_tables(stores):
    return [([s.fact_info(i)[0] for i in range(s.num_facts)],
             [s.fact_info(i)[1] for i in range(s.num_facts)]) for s in stores]


def _shard_stores(wl, n, small_limit=None):
    owner = shard.round_robin_owner(len(wl.fact_lens), n)
    stores = [make_store(wl, small_limit=small_limit, facts=shard.owned_facts(owner, p))
              for p in range(n)]
    return owner, stores


SHAPES = [
    # name, L, H, D, theta, llama3, B
    ("llama-like", 2, 8, 128, 5e5, True, 16),
    ("qwen-like", 2, 4, 128, 1e6, False, 16),
    ("d64-b8", 2, 2, 64, 1e4, False, 8),
]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("n_shards", [1, 3])
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_sharded_view_matches_the_full_store(shape, n_shards, path):
    _need_gpu()
    name, L, H, D, theta, ll3, B_ = shape
    wl = _ragged(synth.Model(name, L, H, D, theta, llama3=ll3), seed=91 + n_shards, B=B_)
    owner, stores = _shard_stores(wl, n_shards, PATHS[path])
    home = stores[0]
    try:
        home.attach_shards([s.arena_ptrs() for s in stores],
                           *shard.global_fact_table(owner, _local_tables(stores)))
        assert home.shard_info() == (n_shards, len(wl.fact_lens))
        assert_parity(oracle_run(wl), gpu_run(wl, store=home))
        home.detach_shards()
        assert home.shard_info() == (0, 0)
    finally:
        for s in stores:
            s.close()


def test_sharded_view_bad_global_id_skips_its_request():
    """An id past the global table is BAD_FACT_ID with its request skipped,
    as on a single store (the oracle on the full store agrees)."""
    _need_gpu()
    wl = _ragged(synth.Model("m", 2, 4, 128, 1e6), seed=95, R=4)
    wl.batch.fact_ids[0] = len(wl.fact_lens)
    owner, stores = _shard_stores(wl, 2)
    try:
        stores[0].attach_shards([s.arena_ptrs() for s in stores],
                                *shard.global_fact_table(owner, _local_tables(stores)))
        o = oracle_run(wl)
        assert o[0] == B.IS_ERR_BAD_FACT_ID
        assert_parity(o, gpu_run(wl, store=stores[0]))
    finally:
        for s in stores:
            s.close()


def test_attach_shards_validates_on_the_host():
    _need_gpu()
    wl = _ragged(synth.Model("m", 1, 2, 64, 1e4), seed=96, R=2, num_facts=6)
    owner, stores = _shard_stores(wl, 2)
    a = [s.arena_ptrs() for s in stores]
    so, off, ln = shard.global_fact_table(owner, _local_tables(stores))
    home = stores[0]
    try:
        bad_shard = so.copy()
        bad_shard[1] = 2
        bad_off = off.copy()
        bad_off[3] = a[int(so[3])][2]  # starts at the plane's end
        bad_len = ln.copy()
        bad_len[0] = 0
        for args in ((a, bad_shard, off, ln), (a, so, bad_off, ln), (a, so, off, bad_len),
                     ([(a[0][0] + 2, a[0][1], a[0][2]), a[1]], so, off, ln),  # unaligned
                     ([(0, a[0][1], a[0][2]), a[1]], so, off, ln)):
            with pytest.raises(B.InjectError) as e:
                home.attach_shards(*args)
            assert e.value.status == B.IS_ERR_INVALID_ARG
        assert home.shard_info() == (0, 0)
        home.attach_shards(a, so, off, ln)
        with pytest.raises(B.InjectError):  # a failed attach keeps the previous view
            home.attach_shards(a, bad_shard, off, ln)
        assert home.shard_info() == (2, len(wl.fact_lens))
        home.detach_shards()
        home.detach_shards()  # no view: nothing to do
    finally:
        for s in stores:
            s.close()
    from synth.device import rope_of
    from kv_cache_injection_gather_b200 import FactStore
    m = wl.model
    host = FactStore(m.num_layers, m.num_kv_heads, m.head_dim, rope_of(m), 64, 4, host_tier=True,
                     hot_capacity_tokens=16)
    try:
        with pytest.raises(B.InjectError) as e:
            host.attach_shards(a, so, off, ln)
        assert e.value.status == B.IS_ERR_NOT_SUPPORTED
        with pytest.raises(B.InjectError) as e:
            host.export()
        assert e.value.status == B.IS_ERR_NOT_SUPPORTED
    finally:
        host.close()


# ------------------------------------------------ two processes, CUDA IPC

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _ipc_wl():
    return _ragged(synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True), seed=97, R=6)


def _ipc_worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        wl = _ipc_wl()
        owner = shard.round_robin_owner(len(wl.fact_lens), world)
        store = make_store(wl, facts=shard.owned_facts(owner, rank), small_limit=0 if rank else None)
        torch.cuda.synchronize()
        grp = shard.FactShardGroup(store, owner)
        res = gpu_run(wl, store=store)  # the whole batch, global ids
        torch.cuda.synchronize()
        info = store.shard_info()
        grp.close()
        store.close()
        np.save(os.path.join(out_dir, f"ipc{rank}.npy"), np.array([(res, info)], dtype=object),
                allow_pickle=True)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
def test_two_processes_read_each_others_shards_through_ipc():
    _need_gpu()
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_ipc_worker, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        outs = [np.load(os.path.join(d, f"ipc{r}.npy"), allow_pickle=True)[0] for r in range(world)]
    wl = _ipc_wl()
    o = oracle_run(wl)
    for res, info in outs:
        assert tuple(info) == (world, len(wl.fact_lens))
        assert_parity(o, res)
