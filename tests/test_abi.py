"""The C-ABI library loads, exports every function include/*.h declares, and
rejects bad arguments on the host before touching a GPU (CPU only)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(is_\w+)\s*\(", text, re.M):
            names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from kv_cache_injection_gather_b200 import build
    return ctypes.CDLL(build.build())


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("is_store_create", "is_store_put_fact", "is_inject_batch", "is_store_destroy",
              "is_last_error", "is_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_binding_names_match_header():
    from kv_cache_injection_gather_b200 import binding
    for n in declared_functions():
        assert hasattr(binding, n), f"binding lacks {n}"


def test_host_validation_without_gpu():
    from kv_cache_injection_gather_b200 import binding as B
    lib = B.lib()
    assert B.status_string(B.IS_ERR_BAD_BLOCK).startswith("block-table")
    out = ctypes.c_void_p()
    assert lib.is_store_create(None, 0, ctypes.byref(out)) == B.IS_ERR_INVALID_ARG
    cfg = B.is_store_config_t(num_layers=1, num_kv_heads=1, head_dim=96, rope_theta=1e4,
                              capacity_tokens=16, max_facts=4)
    assert lib.is_store_create(ctypes.byref(cfg), 0, ctypes.byref(out)) == B.IS_ERR_NOT_SUPPORTED
    cfg.head_dim = 128
    cfg.rope_scaling = B.IS_SCALING_LLAMA3  # factors missing
    assert lib.is_store_create(ctypes.byref(cfg), 0, ctypes.byref(out)) == B.IS_ERR_INVALID_ARG
    cfg.rope_scaling = 0
    cfg.rope_theta = -1.0
    assert lib.is_store_create(ctypes.byref(cfg), 0, ctypes.byref(out)) == B.IS_ERR_INVALID_ARG
    cache = B.is_cache_t()
    assert lib.is_inject_batch(None, 0, None, None, 0, None, None, 1, ctypes.byref(cache), None,
                               0, None) == B.IS_ERR_INVALID_ARG
    assert lib.is_last_error(None, None, None) == B.IS_ERR_INVALID_ARG
    lib.is_store_destroy(None)  # ignored


def test_cache_desc_rejects_what_the_library_cannot_address():
    """Host-side checks of the torch wrapper: caches must be CUDA bf16 5-D
    tensors with a unit innermost stride, K and V alike."""
    import torch
    from kv_cache_injection_gather_b200 import cache_desc
    cpu = torch.zeros(1, 2, 16, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cache_desc(cpu, cpu)  # not on a CUDA device
    with pytest.raises(ValueError):
        cache_desc(cpu.float(), cpu.float())
    with pytest.raises(ValueError):
        cache_desc(cpu[0], cpu[0])  # 4-D
