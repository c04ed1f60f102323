"""The benchmark's command-line contract, checked on CPU: the reference arm
(the CPU oracle) prints one JSON line with the keys of its output contract, only
rank 0 prints under torchrun, too few warm-up steps are refused, and the
GPU arm fails loudly without a CUDA device (no CPU fallback)."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE = [sys.executable, os.path.join(ROOT, "bench.py")]
REF = ["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "llama-single"]


def _run(args, **kw):
    return subprocess.run(args, cwd=ROOT, capture_output=True, text=True, timeout=300, **kw)


def _json_lines(out: str):
    return [json.loads(line) for line in out.splitlines() if line.startswith("{")]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_reference_arm_prints_the_contract_line():
    r = _run(BASE + REF)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert "workload" in d["config"] and d["data"] == "synthetic"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    r = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
              os.path.join(ROOT, "bench.py"), "--gpus", "2"] + REF, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"


def test_too_few_warmup_steps_are_refused():
    r = _run(BASE + ["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0 and "warmup" in (r.stderr + r.stdout)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_gpu_arm_fails_loudly_without_a_gpu():
    r = _run(BASE + ["--steps", "1", "--warmup", "3", "--workload", "llama-single",
                     "--no-cpu-baseline"])
    assert r.returncode != 0
    assert "CUDA device" in (r.stderr + r.stdout)
    assert not _json_lines(r.stdout)


def test_l2_flush_runs_on_any_device():
    """The flush between singly timed steps (a write of twice L2, then a read
    of twice L2) is plain torch work; on the CPU it must run as written."""
    sys.path.insert(0, ROOT)
    import bench
    f = bench.L2Flush("cpu")
    f()
    assert f.buf.numel() == 2 * bench.L2_BYTES and int(f.acc) == 0


def test_launch_count_follows_the_library_path_choice():
    """bench.py counts one kernel per step for a batch the library runs as its
    single kernel and two (plan + inject) otherwise; its limits must be the
    library's (the constants of the kernel header and the host's 32-bit sum
    bound), and its rule the host's: requests <= limit, ids <= 256,
    ids x the longest fact <= 2^31 - 1."""
    import re
    sys.path.insert(0, ROOT)
    import bench
    csrc = os.path.join(ROOT, "kv_cache_injection_gather_b200", "csrc")
    hdr = open(os.path.join(csrc, "inject_kernels.cuh")).read()
    host = open(os.path.join(csrc, "inject_store.cu")).read()
    assert int(re.search(r"constexpr int kSmallRequests = (\d+);", hdr).group(1)) == bench.SMALL_REQUESTS
    assert int(re.search(r"constexpr int kSmallIds = (\d+);", hdr).group(1)) == bench.SMALL_IDS
    assert "kSmallSumLimit = (int64_t(1) << 31) - 1" in host
    assert bench.single_kernel(1, 5, 64)
    assert bench.single_kernel(32, 256, 96)
    assert not bench.single_kernel(33, 5, 64)
    assert not bench.single_kernel(1, 257, 64)
    assert not bench.single_kernel(1, 256, 1 << 23)       # 2^31 tokens by the bound
    assert bench.single_kernel(1, 255, 1 << 23)
    assert not bench.single_kernel(4, 5, 64, limit=0)     # --small-limit 0
    assert bench.single_kernel(8, 5, 64, limit=8) and not bench.single_kernel(9, 5, 64, limit=8)
