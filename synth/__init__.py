"""Seeded synthetic inputs shared by the oracle tests, the CUDA-path tests and bench.py.

This module only draws random numbers and names workload shapes.  It holds none of
the attention arithmetic (no RoPE, no mask, no softmax, no slot mapping), so the
oracle and the CUDA path can both consume it without sharing any of the method.

Value distribution: every Q/K/V element is drawn from N(0, 1) and rounded to
bfloat16, the storage type the Prefix Sliding pages size the KV cache with
(Prefix Sliding 完全拆解, §引子, eq. M_KV uses 2 bytes per element).
Positions are drawn uniformly from the ranges the workloads name.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "normal_bf16",
    "uniform_positions",
    "seed_for",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic workload (head geometry, cache geometry, batch)."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    l_prefix: int
    window: int
    rope_theta: float = 1.0e6
    # decode workloads: positions of the token being decoded
    pos_lo: Optional[int] = None
    pos_hi: Optional[int] = None
    # prefill workloads: sequence length
    seq: Optional[int] = None
    n_layers: int = 1
    group_size: int = 1  # sequences sharing one prompt prefix
    index: int = 0  # 1-based workload index used for the seed


# Workload shapes.  The head geometry is Qwen3-1.7B's (16 query heads, 2 KV heads,
# head_dim 128) or the 7B-class one (28/4/128), as the pages describe the models
# (Prefix Sliding 完全拆解, §引子).
WORKLOADS = {
    "decode_b1_w512": Workload(
        name="decode_b1_w512", batch=1, n_q_heads=16, n_kv_heads=2, head_dim=128,
        l_prefix=100, window=512, pos_lo=100, pos_hi=2147, index=1),
    "decode_b64_w4096": Workload(
        name="decode_b64_w4096", batch=64, n_q_heads=16, n_kv_heads=2, head_dim=128,
        l_prefix=100, window=4096, pos_lo=8192, pos_hi=131072, index=2),
    "prefill_b4_s8192_w2048": Workload(
        name="prefill_b4_s8192_w2048", batch=4, n_q_heads=28, n_kv_heads=4, head_dim=128,
        l_prefix=256, window=2048, seq=8192, index=3),
    "decode_sweep_b256_w8192": Workload(
        name="decode_sweep_b256_w8192", batch=256, n_q_heads=16, n_kv_heads=2, head_dim=128,
        l_prefix=100, window=8192, pos_lo=4096, pos_hi=131072, index=4),
    "decode_stack_l28_b1024_w16384": Workload(
        name="decode_stack_l28_b1024_w16384", batch=1024, n_q_heads=16, n_kv_heads=2,
        head_dim=128, l_prefix=2000, window=16384, pos_lo=32768, pos_hi=262144,
        n_layers=28, index=5),
    # many samples of one prompt (the pages' accuracy tables average 64 samples per
    # problem): 4 prompts x 64 samples, a 2000-token prompt kept as the prefix
    "decode_shared_b256_g64_lp2000_w4096": Workload(
        name="decode_shared_b256_g64_lp2000_w4096", batch=256, n_q_heads=16, n_kv_heads=2,
        head_dim=128, l_prefix=2000, window=4096, pos_lo=8192, pos_hi=131072, group_size=64,
        index=6),
    # a quarter of the truncated-backprop prefill (one sequence of 4096 tokens): small
    # enough for a full profiler capture, still larger than L2
    "prefill_b1_s4096_w2048": Workload(
        name="prefill_b1_s4096_w2048", batch=1, n_q_heads=28, n_kv_heads=4, head_dim=128,
        l_prefix=256, window=2048, seq=4096, index=7),
}


def seed_for(index: int, stream: int = 0) -> int:
    """Seed of workload ``index`` (1000 + index), offset by a sub-stream id."""
    return 1000 + index + 7919 * stream


def _generator(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) samples rounded to bfloat16, drawn from a generator seeded with ``seed``."""
    g = _generator(seed, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def uniform_positions(batch: int, lo: int, hi: int, seed: int, device="cpu") -> torch.Tensor:
    """``batch`` int64 positions drawn uniformly from the closed range [lo, hi]."""
    g = _generator(seed, "cpu")
    p = torch.randint(int(lo), int(hi) + 1, (int(batch),), generator=g, dtype=torch.int64)
    return p.to(device)
