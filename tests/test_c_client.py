"""The boundary is a C ABI: a plain C program (tests/c/abi_c_client.c) built
against include/inject_store.h and libinjectstore.so.  Compiled and linked
on CPU; run on a GPU."""
import os
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def _build(tmp_path):
    from kv_cache_injection_gather_b200 import build
    lib = build.build()
    exe = tmp_path / "abi_c_client"
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c", "abi_c_client.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", os.path.dirname(lib), "-linjectstore", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.dirname(lib)}:{os.path.join(CUDA, 'lib64')}", "-o", str(exe)]
    subprocess.run(cmd, check=True)
    return exe


def test_c_client_compiles_and_links(tmp_path):
    assert _build(tmp_path).exists()


@pytest.mark.gpu
def test_c_client_runs(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([str(_build(tmp_path))], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr + r.stdout
    assert "ok" in r.stdout
