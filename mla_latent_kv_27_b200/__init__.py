"""B200-native MLA decode over a latent KV cache.

The compute lives in libmla.so (hand-written CUDA for sm_100a behind the C ABI in
include/mla.h); this package is its ctypes binding plus a small runner that owns device
buffers (through torch) and issues the four calls of a decode step.  The binding is loaded
on first use; without the built library that first use raises ImportError.
"""
from __future__ import annotations

import importlib

_BINDING_NAMES = {
    "mla_rope_table", "mla_append_workspace_size", "mla_append_cache", "mla_absorb_query",
    "mla_decode_workspace_size", "mla_decode_attention", "mla_output_up", "mla_status_string",
    "mla_check_device_error", "mla_version", "mla_launch_count", "mla_dims", "mla_cache", "MlaError", "lib_handle",
    "MLA_F32", "MLA_BF16", "MLA_FP8_E4M3", "EXPORTED", "mla_decode_attention_noalloc",
    "MLA_NOALLOC_SCRATCH_BYTES",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        mod = importlib.import_module("._binding", __name__)
        return getattr(mod, name)
    raise AttributeError(name)
