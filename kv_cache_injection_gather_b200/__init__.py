"""B200-native retrieve-and-inject: pre-RoPE fact store -> contiguous segment
-> RoPE re-rotation -> paged KV cache scatter, one CUDA library
(libinjectstore.so, C-ABI in include/inject_store.h) for the whole path.

The binding loads the in-tree shared library and raises if it is missing;
there is no CPU or Python fallback for any step of the path.
"""
from . import binding
from .binding import (IS_ERR_BAD_BLOCK, IS_ERR_BAD_FACT_ID, IS_ERR_CAPACITY, IS_ERR_CUDA,
                      IS_ERR_INVALID_ARG, IS_ERR_NOT_SUPPORTED, IS_ERR_OOM, IS_ERR_POSITION,
                      IS_ERR_TIMEOUT, IS_OK, IS_ROPE_INTERLEAVED, IS_ROPE_ROTATE_HALF, InjectError)
from .store import FactStore, RopeConfig, cache_desc

__all__ = ["binding", "FactStore", "RopeConfig", "cache_desc", "InjectError", "IS_OK",
           "IS_ERR_INVALID_ARG", "IS_ERR_BAD_FACT_ID", "IS_ERR_POSITION", "IS_ERR_BAD_BLOCK",
           "IS_ERR_CAPACITY", "IS_ERR_OOM", "IS_ERR_CUDA", "IS_ERR_TIMEOUT",
           "IS_ERR_NOT_SUPPORTED", "IS_ROPE_ROTATE_HALF", "IS_ROPE_INTERLEAVED"]
