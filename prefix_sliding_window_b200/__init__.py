"""Prefix Sliding attention hot path for NVIDIA B200 (sm_100a).

The compute lives in libps.so (C ABI, include/ps.h): the KV append with Continue-PE RoPE,
the split-K decode over the pinned prefix plus the W-slot ring, the full-attention
comparator and the masked (two-level filtered) prefill.  ``binding`` is the thin ctypes
layer over it; ``cache`` allocates the caller-owned buffers with PyTorch.
"""
from . import binding  # noqa: F401
from .binding import (  # noqa: F401
    PsError,
    make_cache,
    make_params,
    ps_decode_attn,
    ps_decode_visible_ranges,
    ps_decode_workspace_bytes,
    ps_full_attn_ref,
    ps_full_attn_workspace_bytes,
    ps_kv_append_rope,
    ps_masked_prefill_attn,
    ps_prefill_plan_tiles,
    ps_prefill_tile_geometry,
    ps_prefill_workspace_bytes,
    ps_version,
)
