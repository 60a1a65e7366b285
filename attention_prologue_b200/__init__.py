"""Gemma 4 decoder attention layer on B200 (sm_100a).

The compute lives in libg4attn.so (hand-written CUDA kernels behind the C ABI
of include/g4attn.h); ``attention_prologue_b200.g4attn`` is its thin ctypes
binding and ``attention_prologue_b200.workloads`` draws seeded synthetic inputs.
"""
from . import g4attn  # noqa: F401  (binding; loads the library lazily)
from .g4attn import (G4AttnError, KVCache, LayerDesc, g4attn_cache_append, g4attn_decode,  # noqa: F401
                     g4attn_decode_workspace_size, g4attn_get_device_status, g4attn_launch_count,
                     g4attn_prefill, g4attn_prefill_workspace_size, g4attn_status_string,
                     g4attn_time_next_attention, make_desc)
