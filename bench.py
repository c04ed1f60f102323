"""Benchmark of the retrieve-and-inject path on B200.

Workload (default): Llama-3.1-8B shapes (32 layers, 8 KV heads, head_dim 128,
theta 5e5 with llama3 scaling), a fact store of 10 000 facts with lengths
uniform in 16..64 tokens (~52 GB of bf16 K+V), and one batch of 100 requests,
each injecting k=50 distinct facts after a 64-token prefix into its own
shuffled 256-block table of a 25 600-block paged cache (block size 16).

One step = one whole batch through the path: segment composition (plan
kernel) + gather, RoPE re-rotation and paged scatter of K and V for every
layer and KV head (inject kernel).  Inputs are synthetic and seeded; the
26 GB read and 26 GB written per step are far larger than the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank is an independent replica
with its own store and batch (requests are independent; no collective on the
data path), so the scaling is weak and the value is the sum over ranks of
tokens divided by the slowest rank's time.  ``--shard heads`` splits the KV
heads of one larger batch over the ranks; ``--shard facts`` splits the facts
over the ranks, each rank injecting 100 requests and reading the facts it
does not hold from the peers' arenas over NVLink inside the inject kernel
(roofline: those bytes at the peer-copy bandwidth).

``--impl reference`` times the CPU oracle (the plain fp64 C definition of the
path) on the host cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "injected KV tokens/s and achieved HBM GB/s (vs ~8 TB/s); per-batch inject µs"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["kv_cache_injection_gather_b200/csrc/inject_kernels.cuh",
                  "kv_cache_injection_gather_b200/csrc/inject_store.cu"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic():
    """DRAM bytes per injected token of the inject kernel from the committed
    ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "inject_kernel_traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except Exception:
        return None, None
    if rec.get("kernel_source_sha256_16") != kernel_source_hash():
        return None, rec
    return float(rec["dram_bytes_per_token"]), rec


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(wl, requests, device=None):
    """Host arrays for the oracle on a subset of requests: the facts those
    requests use (regenerated by the seeded generator) and a compact cache
    holding only their blocks."""
    import oracle
    import synth
    m, b = wl.model, wl.batch
    L, H, D = m.num_layers, m.num_kv_heads, m.head_dim
    used = np.unique(np.concatenate([b.fact_ids[b.req_offsets[r]:b.req_offsets[r + 1]]
                                     for r in requests]))
    remap = {int(f): i for i, f in enumerate(used)}
    st = oracle.Store(L, H, D, int(wl.fact_lens[used].sum()), len(used))
    gen = None
    if device is not None:
        import torch
        gen = torch.empty(L * H * int(wl.fact_lens.max()) * D, dtype=torch.int16,
                          device=f"cuda:{device}")
    for f in used:
        n = int(wl.fact_lens[f])
        if gen is None:
            k, v = synth.fact_kv(wl.seed, int(f), L, H, n, D)
        else:  # the generator's device implementation (same definition, faster)
            cnt = L * H * n * D
            cs = 0
            synth.fill_device(gen.data_ptr(), cnt, wl.seed, synth.fact_stream(int(f), False), 0, cs)
            k = gen[:cnt].cpu().numpy().view(np.uint16).reshape(L, H, n, D)
            synth.fill_device(gen.data_ptr(), cnt, wl.seed, synth.fact_stream(int(f), True), 0, cs)
            v = gen[:cnt].cpu().numpy().view(np.uint16).reshape(L, H, n, D)
        st.put(k, v)
    ids, offs, bts = [], [0], []
    for i, r in enumerate(requests):
        seg = b.fact_ids[b.req_offsets[r]:b.req_offsets[r + 1]]
        ids.extend(remap[int(f)] for f in seg)
        offs.append(len(ids))
        bts.append(np.arange(i * b.max_blocks, (i + 1) * b.max_blocks, dtype=np.int32))
    nb = len(requests) * b.max_blocks
    shape = (L, nb, b.block_size, H, D)
    kc = np.zeros(shape, np.uint16)
    vc = np.zeros(shape, np.uint16)
    inv = oracle.rope_inv_freq(D, m.rope_theta, m.scaling())
    args = (st, inv, np.array(offs, np.int32), np.array(ids, np.int32),
            b.start_pos[list(requests)], np.stack(bts), kc, vc, b.block_size)
    tokens = sum(int(wl.fact_lens[b.fact_ids[b.req_offsets[r]:b.req_offsets[r + 1]]].sum())
                 for r in requests)
    return args, tokens


def time_oracle(args, threads: int) -> float:
    import oracle
    t0 = time.perf_counter()
    rc, _ = oracle.inject_batch(*args, num_threads=threads)
    dt = time.perf_counter() - t0
    if rc != oracle.OK:
        raise RuntimeError(f"oracle status {rc}")
    return dt


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(wl, device, budget_s=15.0):
    """The oracle as it stands, on the host cores, on a bounded sample; also
    its single-thread rate on the first request."""
    import oracle
    threads = oracle.max_threads()
    args, tok = oracle_sample(wl, [0], device)
    dt = time_oracle(args, threads)
    dt1 = time_oracle(args, 1)
    tok1 = tok
    n_req = int(max(1, min(wl.batch.num_requests, budget_s / max(dt, 1e-3))))
    if n_req > 1:
        del args
        args, tok = oracle_sample(wl, list(range(n_req)), device)
        dt = time_oracle(args, threads)
    return {"value": tok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n_req} of {wl.batch.num_requests} requests ({tok} tokens, all "
                      f"{wl.model.num_layers} layers x {wl.model.num_kv_heads} KV heads), "
                      f"{dt:.2f} s",
            "single_thread_value": tok1 / dt1,
            "single_thread_sample": f"request 0 ({tok1} tokens), {dt1:.2f} s",
            "nproc": os.cpu_count(), "cpu_model": cpu_model()}


# ------------------------------------------------------------------ main

WORKLOADS = {
    # name: (description, builder)
    "llama-batch": ("llama3.1-8b-shapes 10k-fact store, 100 requests x k=50, block 16, "
                    "cache 25600 blocks", lambda seed: _synth().llama_batch(seed)),
    "llama-batch-small": ("llama3.1-8b-shapes 500-fact store, 10 requests x k=20, block 16, "
                          "cache 640 blocks (profiling case, ~4 GB on the device)",
                          lambda seed: _synth().llama_batch(seed, num_facts=500, R=10, k=20,
                                                            slots_per_request=1024)),
    "llama-batch-distinct-small": ("llama3.1-8b-shapes 600-fact store, 9 requests x k=22, no fact "
                                   "repeated in the batch, block 16, cache 864 blocks (profiling "
                                   "case for DRAM traffic of the plan + inject path with "
                                   "--small-limit 0, ~5 GB on the device)",
                                   lambda seed: _synth().llama_batch(seed, num_facts=600, R=9, k=22,
                                                                     slots_per_request=1536,
                                                                     distinct_batch=True)),
    "llama-single": ("llama3.1-8b-shapes 10k-fact store, 1 request x k=5, block 16, 64 blocks",
                     lambda seed: _synth().llama_single(seed)),
    "llama-single-small": ("llama3.1-8b-shapes 500-fact store, 1 request x k=5, block 16, 64 blocks "
                           "(profiling case of the single request, ~2.7 GB on the device)",
                           lambda seed: _synth().llama_single(seed, num_facts=500)),
    "offload": ("qwen2.5-7b-shapes store of 16..48-token facts in pinned host memory, HBM hot "
                "set = top 20% by Zipf rank, 100 requests x k=50 drawn Zipf(1.1), block 16",
                lambda seed, n=100_000: _synth().offload(seed, num_facts=n, extra_batches=7)),
    "qwen-sweep": ("qwen2.5-7b-shapes 50k-fact store (lognormal 8..96), R=100 x k=50, block 16",
                   lambda seed: _synth().sweep(_synth().QWEN25_7B, 100, 50, seed)),
    "mistral-sweep": ("mistral-7b-shapes 20k-fact store (lognormal 8..96; capped so store + "
                      "cache fit HBM), R=100 x k=50, block 16",
                      lambda seed: _synth().sweep(_synth().MISTRAL_7B, 100, 50, seed,
                                                  num_facts=20_000)),
}


def _synth():
    import synth
    return synth


def workload_config(wl, name="llama-batch", extra=None):
    m, b = wl.model, wl.batch
    cfg = {"workload": WORKLOADS[name][0],
           "shapes": m.name, "layers": m.num_layers, "kv_heads": m.num_kv_heads,
           "head_dim": m.head_dim,
           "rope": f"theta {m.rope_theta:g}" + (", llama3 scaling (8, 1, 4, 8192)" if m.llama3 else ""),
           "requests": b.num_requests, "k": int(b.req_offsets[1] - b.req_offsets[0]),
           "facts": len(wl.fact_lens),
           "fact_len": {"llama": "uniform 16..64", "offlo": "uniform 16..48"}.get(name[:5],
                                                                                "lognormal 8..96"),
           "store_gb": round(float(wl.fact_lens.sum()) * m.bytes_per_token / 1e9, 2),
           "tokens_per_batch": wl.tokens(), "block_size": b.block_size,
           "num_blocks": b.num_blocks, "start_pos": 64,
           "l2": (f"inputs larger than L2 ({wl.tokens() * m.bytes_per_token / 1e9:.1f} GB read + "
                  f"the same written per step, L2 126 MB)"
                  if wl.tokens() * m.bytes_per_token >= 4 * L2_BYTES else
                  f"{wl.tokens() * m.bytes_per_token / 1e6:.1f} MB read per step, L2 126 MB")}
    if extra:
        cfg.update(extra)
    return cfg


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload][1](0)
    sample_args, tok = oracle_sample(wl, [0], None if not _cuda() else 0)
    import oracle
    threads = oracle.max_threads()
    for _ in range(args.warmup):
        time_oracle(sample_args, threads)
    times = [time_oracle(sample_args, threads) for _ in range(args.steps)]
    total = sum(times)
    value = tok * args.steps / total
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.workload,
                                      {"reference_step": "request 0 of the batch"}),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"request 0 of the batch ({tok} tokens, all layers and "
                                       f"heads) per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def gpu_id(dev, local_rank: int) -> str:
    """nvidia-smi --id for this device (its UUID), else the local rank."""
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(local_rank)


def launch_probe(dev, flush, reps: int = 200) -> float:
    """Microseconds between two CUDA events around the smallest kernel (a
    one-element fill), median of reps timed as the small batches are (each
    after an L2 flush, which the GPU is still running when the events and
    the kernel are queued, so no host time falls between them): the fixed
    cost any single launch timed this way carries on this machine.  Context for
    batches bound by latency, not their denominator."""
    import torch
    t = torch.zeros(1, device=dev)
    pairs = []
    for _ in range(reps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        t.fill_(1.0)
        e1.record()
        pairs.append((e0, e1))
    torch.cuda.synchronize(dev)
    return float(np.median([a.elapsed_time(b) * 1e3 for a, b in pairs]))


def copy_probe(dev, elems: int = 1 << 30, reps: int = 10):
    """Device copy bandwidth on this machine now (read + write bytes / time): the
    best of reps single copies (the kind of figure the measured peak is) and
    the average of ~0.8 s of copies back to back (a sustained figure, under
    the same power cap as a long timed region).  Context for the roofline
    fraction, not its denominator."""
    import torch
    a = torch.empty(elems, dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    b.copy_(a)
    best = float("inf")
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        b.copy_(a)
        e1.record()
        torch.cuda.synchronize(dev)
        best = min(best, e0.elapsed_time(e1))
    # sustained: back to back for about as long as a timed region
    n = max(1, int(800.0 / best))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        b.copy_(a)
    e1.record()
    torch.cuda.synchronize(dev)
    sustained = n * 2 * elems * 2 / (e0.elapsed_time(e1) / 1e3) / 1e9
    del a, b
    torch.cuda.empty_cache()
    return 2 * elems * 2 / (best / 1e3) / 1e9, sustained


L2_BYTES = 126 * (1 << 20)


class L2Flush:
    """Writes a buffer twice the size of L2 on the launching stream, then
    reads another one of that size, so the next step's reads start from HBM
    (for steps whose reads fit in L2) and the write's dirty lines have gone
    back to HBM before the step starts, as in a cache that was flushed and
    invalidated -- otherwise a step timed alone pays for writing back
    126 MB that are not its own."""

    def __init__(self, dev):
        import torch
        self.buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.rd = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
        self.acc = torch.zeros((), dtype=torch.int64, device=dev)

    def __call__(self):
        import torch
        self.buf.zero_()
        torch.sum(self.rd, dim=0, dtype=torch.int64, out=self.acc)


def timed_steps(step, steps, stream, flush=None) -> float:
    """Milliseconds of `steps` calls of step() on `stream`, CUDA events: one
    pair around all of them back to back, or, with `flush`, a flush before
    each step and a pair around each step alone (the flush not counted)."""
    import torch
    if flush is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)
    pairs = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        pairs.append((a, b))
    pairs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs)


def h2d_probe(dev, nbytes: int = 1 << 30, reps: int = 5) -> float:
    """Pinned host -> device copy bandwidth (GB/s), CUDA events."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        d.copy_(h, non_blocking=True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        d.copy_(h, non_blocking=True)
    e1.record()
    torch.cuda.synchronize(dev)
    return reps * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9


def peer_probe(dev, world: int, nbytes: int = 1 << 30, reps: int = 5) -> float:
    """Per-GPU receive bandwidth from the peers (GB/s), measured in this run:
    an all-to-all of nbytes per rank, in which every GPU takes (N-1)/N of its
    bytes from the other GPUs at once -- the pattern of a fact-sharded batch,
    whose rows come from every peer's arenas.  Timed with CUDA events on the
    current stream (wall clock on CPU ranks), max over ranks."""
    import torch
    import torch.distributed as dist
    cuda = torch.device(dev).type == "cuda"
    n = (nbytes // (4 * world)) * world
    src = torch.ones(n, dtype=torch.float32, device=dev)
    dst = torch.empty_like(src)
    dist.all_to_all_single(dst, src)  # warm-up (connections)
    dist.barrier()
    if cuda:
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
    t0 = time.perf_counter()
    for _ in range(reps):
        dist.all_to_all_single(dst, src)
    if cuda:
        e1.record()
        torch.cuda.synchronize(dev)
        sec = e0.elapsed_time(e1) / 1e3
    else:
        sec = time.perf_counter() - t0
    (sec,) = max_over_ranks([sec], world)
    return reps * (n * 4) * (world - 1) / world / sec / 1e9


def max_over_ranks(values, world):
    """Element-wise max of per-rank numbers (timings) over all ranks."""
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.is_initialized() and \
        dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def run_offload(args, rank, world, local_rank):
    """Host-tier store: a stream of 8 different Zipf batches, cycled.  Static
    hot set (top 20% by rank, device-index entry point) or LRU hot set (same
    HBM capacity in 48-token slots, host-index entry point: each batch promotes
    its cold facts as it reads them; with --lru-prefetch each call also starts
    the next batch's cold facts while it runs)."""
    import psutil
    import torch

    import synth
    from synth.device import make_cache, make_store
    from kv_cache_injection_gather_b200 import binding as B

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    n_facts = 100_000
    avail = psutil.virtual_memory().available
    while n_facts * 32 * synth.QWEN25_7B.bytes_per_token > 0.6 * avail and n_facts > 5_000:
        n_facts = int(n_facts * 0.8)
    wl = WORKLOADS["offload"][1](rank, n_facts)
    m, b0 = wl.model, wl.batch
    hot = wl.notes["hot"]
    hot_tokens = int(wl.fact_lens[hot].sum())
    store = make_store(wl, on_device_gen=True, device=local_rank, host_tier=True,
                       hot_capacity_tokens=hot_tokens)
    lru = args.hot_policy == "lru"
    if lru:
        store.set_hot_policy(True, 48)  # slots of the longest fact, same HBM tokens
    else:
        store.set_hot(hot)
    batches = [b0] + [synth.Batch(b0.req_offsets, ids, b0.start_pos, b0.block_tables,
                                  b0.block_size, b0.num_blocks) for ids in wl.notes["more_ids"]]
    ntoks = [int(wl.fact_lens[bb.fact_ids].sum()) for bb in batches]
    kcache, vcache, desc = make_cache(wl, device=local_rank, fill=False)
    stream = torch.cuda.current_stream(dev)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    dvc = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)  # noqa: E731
    host_b = [(pin(bb.req_offsets), pin(bb.fact_ids), pin(bb.start_pos), pin(bb.block_tables))
              for bb in batches]
    dev_b = [(dvc(bb.req_offsets), dvc(bb.fact_ids), dvc(bb.start_pos), dvc(bb.block_tables))
             for bb in batches]
    d_slots = torch.empty(max(ntoks), dtype=torch.int64, device=dev)
    h_slots = torch.empty(max(ntoks), dtype=torch.int64).pin_memory()

    def step(i):
        j = i % len(batches)
        if lru:
            # with --lru-prefetch, the next batch's cold facts move into HBM while this one runs
            rc = store.inject_host(*host_b[j], desc, h_slots[:ntoks[j]], stream.cuda_stream,
                                   next_fact_ids=(host_b[(i + 1) % len(batches)][1]
                                                  if args.lru_prefetch else None))
            if rc != 0:
                raise RuntimeError(f"inject_host failed: {B.status_string(rc)}")
        else:
            store.inject(*dev_b[j], desc, d_slots[:ntoks[j]], stream.cuda_stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    st0 = store.lru_stats() if lru else None
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_id(dev, local_rank))
    clocks.start()
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    rc, _ = store.last_error()
    if rc != 0:
        raise RuntimeError(f"inject failed: {B.status_string(rc)}")
    st1 = store.lru_stats() if lru else None
    store.set_timing(True)
    store.kernel_time()
    for i in range(args.steps):
        step(args.warmup + i)
    torch.cuda.synchronize(dev)
    kern_ms, kern_n = store.kernel_time()
    store.set_timing(False)
    ms, kern_avg_ms = max_over_ranks([ms, kern_ms / max(kern_n, 1)], world)
    tok_run = sum(ntoks[(args.warmup + i) % len(batches)] for i in range(args.steps))
    value = world * tok_run / (ms / 1e3)
    bpt = m.bytes_per_token
    peak, peak_kind = hbm_peak()
    link = h2d_probe(dev)
    if lru:
        prom_tok = st1["promoted_tokens"] - st0["promoted_tokens"]
        link_bytes = prom_tok * bpt
        hbm_bytes = (2 * tok_run + prom_tok) * bpt
        t_min = max(link_bytes / (link * 1e9), hbm_bytes / (peak * 1e9))
        hits = st1["hits"] - st0["hits"]
        misses = st1["misses"] - st0["misses"]
        detail = {"id_hit_fraction": hits / max(hits + misses, 1),
                  "promoted_tokens_per_step": prom_tok / args.steps}
        measured_s = ms / 1e3
    else:
        is_hot = np.zeros(len(wl.fact_lens), bool)
        is_hot[hot] = True
        t_min, link_bytes, hit_tok = 0.0, 0, 0
        for i in range(args.steps):
            bb = batches[(args.warmup + i) % len(batches)]
            per = wl.fact_lens[bb.fact_ids].astype(np.int64)
            hit = int(per[is_hot[bb.fact_ids]].sum())
            miss_b = (int(per.sum()) - hit) * bpt
            t_min += max(miss_b / (link * 1e9), (hit + int(per.sum())) * bpt / (peak * 1e9))
            link_bytes += miss_b
            hit_tok += hit
        hbm_bytes = (hit_tok + tok_run) * bpt
        detail = {"hit_token_fraction": hit_tok / max(tok_run, 1)}
        measured_s = kern_avg_ms * args.steps / 1e3
    algo = 2 * tok_run * bpt
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, "offload", {
            "facts_note": f"{n_facts} facts (host memory available {avail / 1e9:.0f} GB)",
            "hot_policy": args.hot_policy, "hot_tokens_per_plane": hot_tokens,
            "prefetch": ("each batch's call starts the next batch's cold facts over the host link "
                         "while the batch runs" if lru and args.lru_prefetch else None),
            "batches": f"{len(batches)} Zipf batches cycled", "parallelism": f"replicas x{world}"}),
        "us_per_batch": ms / args.steps * 1e3, "kernel_us": kern_avg_ms * 1e3, "clocks": clk,
        "gpu_launches": (4 if lru else 2) * args.steps,
        "roofline": {"bound": "host_link+hbm", "achieved": algo / measured_s / 1e9,
                     "peak": algo / t_min / 1e9, "unit": "GB/s", "frac": t_min / measured_s,
                     "peak_source": f"pinned H2D probe {link:.1f} GB/s for {link_bytes / 1e9:.2f} GB "
                                    f"over the host link; {peak_kind} hbm_gbs {peak} for "
                                    f"{hbm_bytes / 1e9:.1f} GB in HBM; per step the slower bounds",
                     "timed": "whole step (promotion + plan + inject)" if lru else
                              "inject kernel (plan excluded)", **detail},
        "cpu_baseline": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    store.close()
    return 0


SWEEP_R = (1, 16, 100, 256)
SWEEP_K = (5, 10, 20, 50)


SMALL_REQUESTS, SMALL_IDS = 32, 256  # the library's single-kernel limits (default)


def single_kernel(R, num_ids, longest, limit=None):
    """Whether the library runs a batch as its one fused kernel: at most
    `limit` (default 32) requests and 256 ids, 32-bit token sums."""
    lim = SMALL_REQUESTS if limit is None else limit
    return R <= lim and num_ids <= SMALL_IDS and num_ids * longest < 2 ** 31


def run_sweep(args, rank, world, local_rank):
    """Every (R, k) point of the Mistral / Qwen sweep with one store: the
    sweep's fact lengths come first from its seed, so every point draws from
    the same pool.  One JSON line per point (rank 0; each rank runs the
    grid on its own GPU as a replica).  Points whose reads fit in a few L2s
    are timed step by step with an L2 flush between steps."""
    import torch

    from synth.device import batch_tensors, make_cache, make_store
    from kv_cache_injection_gather_b200 import binding as B
    S = _synth()
    if args.workload not in ("qwen-sweep", "mistral-sweep"):
        raise SystemExit("--sweep is defined for qwen-sweep and mistral-sweep")
    model, nf = (S.QWEN25_7B, 50_000) if args.workload == "qwen-sweep" else (S.MISTRAL_7B, 20_000)
    dev = torch.device("cuda", local_rank)
    base = S.sweep(model, 1, 5, rank, num_facts=nf)
    store = make_store(base, on_device_gen=True, device=local_rank)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()
    flusher = L2Flush(dev)
    for R in SWEEP_R:
        for k in SWEEP_K:
            wl = S.sweep(model, R, k, rank, num_facts=nf)
            if not np.array_equal(wl.fact_lens, base.fact_lens):
                raise RuntimeError("sweep points must share the fact pool")
            kc, vc, desc = make_cache(wl, device=local_rank, fill=False)  # kc, vc live for the point
            ro, ids, sp, bt = batch_tensors(wl.batch, local_rank)
            n_tok = wl.tokens()
            slots = torch.empty(max(n_tok, 1), dtype=torch.int64, device=dev)

            def step():
                store.inject(ro, ids, sp, bt, desc, slots[:n_tok], stream.cuda_stream)

            for _ in range(args.warmup):
                step()
            rc, _ = store.last_error()
            if rc != 0:
                raise RuntimeError(f"sweep R={R} k={k}: {B.status_string(rc)}")
            read_bytes = n_tok * model.bytes_per_token
            flush = flusher if read_bytes < 4 * L2_BYTES else None
            est_s = 2 * read_bytes / (peak * 1e9) + 15e-6
            steps = int(min(2000, max(20, 0.3 / est_s)))
            torch.cuda.synchronize(dev)
            ms = timed_steps(step, steps, stream, flush)
            store.set_timing(True)
            store.kernel_time()
            for _ in range(steps):
                if flush is not None:
                    flush()
                step()
            kern_ms, kern_n = store.kernel_time()
            store.set_timing(False)
            kern = kern_ms / max(kern_n, 1)
            extra = {}
            if single_kernel(R, len(wl.batch.fact_ids), int(wl.fact_lens.max())):
                # the same batch through the plan + inject kernels, for the path choice
                store.set_small_batch_limit(0)
                for _ in range(args.warmup):
                    step()
                torch.cuda.synchronize(dev)
                ms2 = timed_steps(step, steps, stream, flush)
                store.set_small_batch_limit(SMALL_REQUESTS)
                extra = {"path": "single kernel", "two_kernel_us_per_batch": ms2 / steps * 1e3}
            if rank == 0:
                print(json.dumps({
                    "metric": METRIC, "workload": WORKLOADS[args.workload][0].split(",")[0],
                    "shapes": model.name, "requests": R, "k": k, "tokens_per_batch": n_tok,
                    "steps": steps, "l2": "flushed before every step" if flush else "reads > 4x L2",
                    "us_per_batch": ms / steps * 1e3, "tokens_per_s": n_tok / (ms / steps / 1e3),
                    "kernel_us": kern * 1e3,
                    "kernel_frac_of_peak": 2 * read_bytes / (kern / 1e3) / 1e9 / peak,
                    "peak_gbs": peak, "peak_source": f"{peak_kind} hbm_gbs", **extra}), flush=True)
            del kc, vc, desc, slots
            torch.cuda.empty_cache()
    store.close()
    return 0


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from synth.device import batch_tensors, make_cache, make_store
    from kv_cache_injection_gather_b200 import binding as B

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the inject path has no CPU fallback)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.workload == "offload":
        return run_offload(args, rank, world, local_rank)
    if args.sweep:
        return run_sweep(args, rank, world, local_rank)
    extra_cfg = {}
    heads = None
    owner = None
    if args.shard == "facts":
        # Fact shards: one fact pool and one batch of 100 requests for every
        # rank; rank p holds the facts g with g % N == p and injects the whole
        # batch (global ids) into its own cache, reading the other ranks'
        # facts from their arenas over NVLink inside the inject kernel.
        from kv_cache_injection_gather_b200 import shard
        if args.workload not in ("llama-batch", "llama-batch-small"):
            raise SystemExit("--shard facts is defined for the llama-batch workloads")
        wl = WORKLOADS[args.workload][1](0)
        owner = shard.round_robin_owner(len(wl.fact_lens), world)
        extra_cfg["facts_per_rank"] = int((owner == rank).sum())
    elif args.shard == "heads":
        # KV-head shards (tensor-parallel serving): every rank holds heads
        # [h0, h1) of every fact and of the cache and injects the same batch of
        # 100 x world requests; per-GPU bytes stay those of the 1-GPU batch.
        import synth
        from kv_cache_injection_gather_b200 import shard
        if args.workload != "llama-batch":
            raise SystemExit("--shard heads is defined for the llama-batch workload")
        wl = synth.llama_batch(0, R=100 * world)
        heads = shard.head_shard(wl.model.num_kv_heads, world, rank)
        extra_cfg["kv_heads_per_rank"] = heads[1] - heads[0]
    else:
        wl = WORKLOADS[args.workload][1](rank)
    store = make_store(wl, on_device_gen=True, device=local_rank, heads=heads,
                       facts=None if owner is None else shard.owned_facts(owner, rank),
                       small_limit=args.small_limit)
    group = None
    if owner is not None:
        if world > 1:
            group = shard.FactShardGroup(store, owner)
        else:
            info = [store.fact_info(i) for i in range(store.num_facts)]
            store.attach_shards([store.arena_ptrs()], *shard.global_fact_table(
                owner, [([o for o, _ in info], [n for _, n in info])]))
    m, b = wl.model, wl.batch
    if heads is not None:
        m = synth.Model(m.name, m.num_layers, heads[1] - heads[0], m.head_dim, m.rope_theta, m.llama3)
    kcache, vcache, desc = make_cache(wl, device=local_rank, fill=False, head_major=args.head_major,
                                      num_kv_heads=None if heads is None else heads[1] - heads[0])
    extra_cfg["cache_layout"] = "[L][num_blocks][H][B][D]" if args.head_major else "[L][num_blocks][B][H][D]"
    extra_cfg["path"] = ("single fused kernel" if single_kernel(
        b.num_requests, len(b.fact_ids), int(wl.fact_lens.max()), args.small_limit)
        else "plan + inject kernels")  # the kernel the roofline times
    copy_ref, copy_sus = copy_probe(dev)
    # every rank takes part in the same collectives, in the same order
    peer_gbs = peer_probe(dev, world) if (owner is not None and world > 1) else None
    ro, ids, sp, bt = batch_tensors(b, local_rank)
    n_tok = wl.tokens()
    slots = torch.empty(n_tok, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        store.inject(ro, ids, sp, bt, desc, slots, stream.cuda_stream)

    for _ in range(args.warmup):
        step()
    rc, _ = store.last_error()
    if rc != 0:
        raise RuntimeError(f"inject failed during warm-up: {B.status_string(rc)}")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # Steps whose reads fit in a few L2s would re-read cached rows: flush L2
    # before each of them and time each step alone.
    read_bytes = n_tok * m.bytes_per_token
    flush = L2Flush(dev) if read_bytes < 4 * L2_BYTES else None
    if flush is not None:
        extra_cfg["l2"] = (f"flushed before every step (a {2 * L2_BYTES >> 20} MiB write, then a "
                           f"{2 * L2_BYTES >> 20} MiB read so its dirty lines are back in HBM; not "
                           f"timed): {read_bytes / 1e6:.1f} MB read per step, L2 126 MB")

    clocks = ClockSampler(gpu_id(dev, local_rank))
    # ---- device-resident timed region (the value)
    barrier()
    clocks.start()
    ms = timed_steps(step, args.steps, stream, flush)
    barrier()
    clk = clocks.stop()
    rc, _ = store.last_error()
    if rc != 0:
        raise RuntimeError(f"inject failed: {B.status_string(rc)}")

    # ---- the inject kernel alone, for the roofline: the library brackets it
    # with CUDA events on the launching stream (same steps, plan excluded)
    store.set_timing(True)
    store.kernel_time()  # reset
    barrier()
    for _ in range(args.steps):
        if flush is not None:
            flush()
        step()
    barrier()
    kern_ms, kern_n = store.kernel_time()
    store.set_timing(False)

    # ---- end to end through the host entry point: index arrays from pinned
    # host memory in, slot mapping and status back to pinned host memory
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    h_ro, h_ids, h_sp, h_bt = pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos), pin(b.block_tables)
    h_slots = torch.empty(n_tok, dtype=torch.int64).pin_memory()
    h2d = sum(t.numel() * 4 for t in (h_ro, h_ids, h_sp, h_bt))
    d2h = n_tok * 8 + 16
    for _ in range(max(1, args.warmup // 2)):
        store.inject_host(h_ro, h_ids, h_sp, h_bt, desc, h_slots, stream.cuda_stream)
    barrier()

    def host_step():
        rc = store.inject_host(h_ro, h_ids, h_sp, h_bt, desc, h_slots, stream.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"inject_host failed: {B.status_string(rc)}")

    e2e_ms = timed_steps(host_step, args.steps, stream, flush)
    barrier()

    # ---- max over ranks
    ms, e2e_ms, kern_avg_ms = max_over_ranks([ms, e2e_ms, kern_ms / max(kern_n, 1)], world)
    ms_step = ms / args.steps
    tokens_all = n_tok * (1 if heads is not None else world)
    value = tokens_all / (ms_step / 1e3)
    algo_bytes = n_tok * 2 * m.bytes_per_token   # read K+V + write K+V
    peak, peak_kind = hbm_peak()
    achieved = algo_bytes / (kern_avg_ms / 1e3) / 1e9
    single = single_kernel(b.num_requests, len(b.fact_ids), int(wl.fact_lens.max()), args.small_limit)
    traffic_pt, rec = recorded_traffic()
    if args.workload != "llama-batch" or args.head_major or owner is not None:
        traffic_pt = None  # the committed counters are for the benchmark workload
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{peak_kind} hbm_gbs",
                "same_box_copy_gbs": copy_ref, "frac_of_same_box_copy": achieved / copy_ref,
                "same_box_sustained_copy_gbs": copy_sus,
                "frac_of_same_box_sustained_copy": achieved / copy_sus,
                "traffic": None if traffic_pt is None else traffic_pt * n_tok,
                "algorithmic_bytes": algo_bytes,
                "kernel": ("small_inject_kernel (its in-kernel plan included)" if single else
                           "inject_kernel (plan_kernel excluded)")}
    if flush is not None:
        # a batch this small is timed alone: what an empty kernel costs so
        roofline["empty_kernel_us"] = launch_probe(dev, flush)
    if owner is not None and world > 1:
        # Peer reads: rows of facts other ranks own cross NVLink once; the
        # bound is those bytes at the peer bandwidth measured in this run.
        ids_all = b.fact_ids
        remote_tok = int(wl.fact_lens[ids_all[owner[ids_all] != rank]].sum())
        link_bytes = remote_tok * m.bytes_per_token
        link = link_bytes / (kern_avg_ms / 1e3) / 1e9
        roofline = {"bound": "nvlink", "achieved": link, "peak": peer_gbs,
                    "unit": "GB/s", "frac": link / peer_gbs,
                    "peak_source": f"in-run peer probe: NCCL all-to-all of 1 GiB per rank, "
                                   f"per-GPU receive bandwidth over {world} GPUs (max over ranks)",
                    "link_bytes": link_bytes, "hbm_achieved_gbs": achieved,
                    "hbm_frac": achieved / peak, "traffic": None, "algorithmic_bytes": algo_bytes,
                    "kernel": "inject_kernel (plan_kernel excluded)"}
    baseline = cpu_baseline(wl, local_rank) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if group is not None:
        group.close()
    if rank != 0:
        store.close()
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, args.workload,
                                  dict(extra_cfg, parallelism=(
                                      f"kv-head shards x{world}" if heads is not None else
                                      f"fact shards x{world} (peer reads over NVLink)" if owner is not None
                                      else f"replicas x{world}"))),
        "us_per_batch": ms_step * 1e3,
        "gbs_per_gpu": algo_bytes / (ms_step / 1e3) / 1e9,
        "kernel_us": kern_avg_ms * 1e3,
        "clocks": clk,
        "e2e": {"value": tokens_all / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        # the library's kernels per step: one fused kernel for a batch the
        # single-kernel path takes, else the plan and the inject kernel
        "gpu_launches": (1 if single_kernel(b.num_requests, len(b.fact_ids), int(wl.fact_lens.max()),
                                            args.small_limit) else 2) * args.steps,
        "roofline": roofline,
        "cpu_baseline": baseline,
    }
    print(json.dumps(line), flush=True)
    store.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--hot-policy", choices=["static", "lru"], default="static",
                    help="offload workload: static top-20%% hot set or LRU promotion")
    ap.add_argument("--lru-prefetch", action="store_true",
                    help="offload workload, LRU: each call also prefetches the next batch's cold facts")
    ap.add_argument("--shard", choices=["replicas", "heads", "facts"], default="replicas",
                    help="multi-GPU: independent replicas (default), KV-head shards of one "
                         "batch of 100 x N requests (both weak scaling, no collective), or fact "
                         "shards (each rank holds 1/N of the facts and injects 100 requests, "
                         "reading the rest from peers over NVLink)")
    ap.add_argument("--small-limit", type=int, default=None,
                    help="batches of up to this many requests (0..32, default 32) run as the "
                         "single fused kernel; 0: always the plan + inject kernels")
    ap.add_argument("--sweep", action="store_true",
                    help="qwen-sweep / mistral-sweep: every point of R in {1, 16, 100, 256} x k in "
                         "{5, 10, 20, 50} with one store, one JSON line per point")
    ap.add_argument("--head-major", action="store_true",
                    help="cache layout [L][num_blocks][H][B][D] instead of [L][num_blocks][B][H][D]")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama-batch",
                    help="llama-batch is the benchmark; the others are smaller cases for "
                         "profiling and latency")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    try:
        if args.impl == "reference":
            rc = run_reference(args, rank, world)
        else:
            rc = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
