"""Caller-owned buffers for libps, allocated with PyTorch (device memory only, no compute).

PrefixSlidingCache: the bounded per-sequence KV store of the Prefix Sliding method, a
pinned prefix region [B, Hkv, L_prefix, D] plus a W-slot ring [B, Hkv, W, D] (bf16).  At
most L_prefix + W tokens per sequence are held ("Prefix Sliding 完全拆解", §核心机制,
eq. L_total).

LinearCache: the full-attention comparator's cache [B, Hkv, Lmax, D], passed to the
library as a prefix-only store with l_prefix = Lmax.
"""
from __future__ import annotations

import math

import torch

from .binding import PsKVCache, make_cache, make_params


def _alloc(shape, device, fill):
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if fill is not None:
        t.fill_(fill)
    return t


class PrefixSlidingCache:
    def __init__(self, batch: int, n_kv_heads: int, l_prefix: int, window: int,
                 head_dim: int = 128, device="cuda", fill=0.0):
        self.batch, self.n_kv_heads, self.head_dim = batch, n_kv_heads, head_dim
        self.l_prefix, self.window = l_prefix, window
        if l_prefix > 0:
            self.k_prefix = _alloc((batch, n_kv_heads, l_prefix, head_dim), device, fill)
            self.v_prefix = _alloc((batch, n_kv_heads, l_prefix, head_dim), device, fill)
        else:
            self.k_prefix = self.v_prefix = None
        self.k_ring = _alloc((batch, n_kv_heads, window, head_dim), device, fill)
        self.v_ring = _alloc((batch, n_kv_heads, window, head_dim), device, fill)
        self._struct = make_cache(self.k_prefix, self.v_prefix, self.k_ring, self.v_ring, batch)

    @property
    def struct(self) -> PsKVCache:
        return self._struct

    def nbytes(self) -> int:
        per = self.batch * self.n_kv_heads * self.head_dim * 2 * 2
        return per * (self.l_prefix + self.window)


class LinearCache:
    def __init__(self, batch: int, n_kv_heads: int, lmax: int, head_dim: int = 128,
                 device="cuda", fill=0.0):
        self.batch, self.n_kv_heads, self.head_dim, self.lmax = batch, n_kv_heads, head_dim, lmax
        self.k = _alloc((batch, n_kv_heads, lmax, head_dim), device, fill)
        self.v = _alloc((batch, n_kv_heads, lmax, head_dim), device, fill)
        self._struct = make_cache(self.k, self.v, None, None, batch)

    @property
    def struct(self) -> PsKVCache:
        return self._struct

    def params(self, n_q_heads: int, rope_theta: float = 1.0e6):
        """Parameters that make ps_kv_append_rope fill this linear cache."""
        return make_params(n_q_heads, self.n_kv_heads, self.head_dim, self.lmax, 1, rope_theta)


def default_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)
