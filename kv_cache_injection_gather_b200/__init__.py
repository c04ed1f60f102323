"""B200-native retrieve-and-inject: pre-RoPE fact store -> contiguous segment
-> RoPE re-rotation -> paged KV cache scatter, one CUDA library
(libinjectstore.so, C-ABI in include/inject_store.h) for the whole path.

The library is loaded on first use of anything but ``build``; a missing or
stale library raises there.  There is no CPU or Python fallback for any step
of the path.
"""
import importlib

_LAZY = {
    "binding": ("binding", None),
    "FactStore": ("store", "FactStore"),
    "RopeConfig": ("store", "RopeConfig"),
    "cache_desc": ("store", "cache_desc"),
    "InjectError": ("binding", "InjectError"),
}
_CONSTS = ("IS_OK", "IS_ERR_INVALID_ARG", "IS_ERR_BAD_FACT_ID", "IS_ERR_POSITION",
           "IS_ERR_BAD_BLOCK", "IS_ERR_CAPACITY", "IS_ERR_OOM", "IS_ERR_CUDA", "IS_ERR_TIMEOUT",
           "IS_ERR_NOT_SUPPORTED", "IS_ROPE_ROTATE_HALF", "IS_ROPE_INTERLEAVED")

__all__ = list(_LAZY) + list(_CONSTS)


def __getattr__(name):
    if name in _LAZY:
        mod, attr = _LAZY[name]
        m = importlib.import_module(f"{__name__}.{mod}")
        return m if attr is None else getattr(m, attr)
    if name in _CONSTS:
        return getattr(importlib.import_module(f"{__name__}.binding"), name)
    raise AttributeError(name)
