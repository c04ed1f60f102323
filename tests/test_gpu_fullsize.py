"""Full-size parity on the benchmark's workload, in the benchmark's launch
configuration: Llama-3.1-8B shapes (32 layers, 8 KV heads, D=128, llama3
RoPE scaling), 10k facts of 16-64 tokens (about 52 GB of store), 100
requests x k=50 distinct facts after a 64-token prefix, 25 600-block cache
(53.7 GB of K and V), token-major and head-major.  The oracle cannot hold
the whole cache, so fullsize_check streams the batch request by request:
every slot, every row -- each (token, layer, head) row of K and V against
the oracle's injection of that request from regenerated inputs -- and every
untouched element.
"""
from __future__ import annotations

import pytest
import torch

import synth
from fullsize_check import check_full_size
from synth.device import make_store

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def llama_store():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    free, _ = torch.cuda.mem_get_info()
    wl = synth.llama_batch(0)
    m, b = wl.model, wl.batch
    need = (int(wl.fact_lens.sum()) + b.num_blocks * b.block_size) * m.bytes_per_token
    if free < need + (8 << 30):
        pytest.skip(f"needs {need / 1e9:.0f} GB free on the device")
    store = make_store(wl, on_device_gen=True)
    yield wl, store
    store.close()


@pytest.mark.parametrize("head_major", [False, True], ids=["token-major", "head-major"])
def test_llama_batch_full_size(llama_store, head_major):
    wl, store = llama_store
    check_full_size(wl, store, head_major=head_major)
