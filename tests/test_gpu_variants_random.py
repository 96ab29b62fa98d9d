"""GPU parity of the decode variants on seeded random geometries against the float64 oracle.

The same checks as the variants' own test files, on drawn geometries instead of hand-picked
ones ("Prefix Sliding 完全拆解": §位置编码 for Reset PE, §核心机制 eq. A(i) for the visible
set, the paged and shared-prefix stores of the vLLM deployment the page describes):
* Reset PE: every output row against the oracle's literal Reset PE (renumber, rotate,
  attend);
* paged store: blocks scattered in a random order, some sequences sharing their prompt's
  blocks, against the oracle and against the contiguous store's decode;
* shared-prefix decode: groups of sequences on one prompt, against the oracle and the plain
  decode of the same histories.
Positions are drawn around the prefix end, the exact cap L_prefix + W and the first
eviction.
"""
import math

import numpy as np
import pytest

from prefix_sliding_window_b200 import binding as B
from tests.test_gpu_paged import _paged_case
from tests.test_gpu_reset_pe import _check_oracle, _decode, _setup
from tests.test_gpu_shared_prefix import _shared_prefix_case

pytestmark = pytest.mark.gpu

D = 128
GROUPINGS = [(16, 2), (8, 8), (28, 4), (4, 1), (24, 3), (8, 1)]


def _positions(rng, lp, w, n, spread):
    """n positions: a few on the eq. A(i) boundaries, the rest uniform in [0, spread)."""
    edges = [lp - 1, lp, lp + w - 1, lp + w, lp + w + 1, lp + 2 * w + 3]
    pos = [int(rng.integers(0, spread)) for _ in range(n)]
    for i in range(min(n, 3)):
        pos[i] = edges[int(rng.integers(0, len(edges)))]
    return [max(0, p) for p in pos]


@pytest.mark.parametrize("seed", range(8))
def test_reset_pe_random_geometry(cuda_device, seed):
    rng = np.random.default_rng(6100 + seed)
    hq, hkv = GROUPINGS[seed % len(GROUPINGS)]
    lp = int(rng.choice([0, 1, 64, 100, int(rng.integers(0, 300))]))
    w = int(rng.choice([1, 63, 64, 256, int(rng.integers(1, 700))]))
    # even cases: far positions (few sequences: the oracle holds each whole history)
    far = seed % 2 == 0
    spread = 70000 if far else 3 * (lp + w) + 100
    positions = _positions(rng, lp, w, int(rng.integers(1, 5 if far else 10)), spread)
    params, cache, pos, q, raw, st = _setup(cuda_device, hq, hkv, lp, w, positions,
                                            seed=6200 + 10 * seed)
    out, lse = _decode(B.ps_decode_attn_reset_pe, params, cache, q, pos, st)
    _check_oracle(out, lse, raw, positions, lp, w, 1 / math.sqrt(D), f"reset seed={seed}")


@pytest.mark.parametrize("seed", range(6))
def test_paged_random_geometry(cuda_device, seed):
    rng = np.random.default_rng(6300 + seed)
    hq, hkv = GROUPINGS[seed % len(GROUPINGS)]
    lp = int(rng.choice([1, 63, 64, 65, int(rng.integers(1, 200))]))
    w = 64 * int(rng.integers(1, 9))
    bn = int(rng.integers(2, 11))
    share = int(rng.integers(1, bn + 1))
    positions = _positions(rng, lp, w, bn, 3 * (lp + w) + 100)
    _paged_case(cuda_device, lp, w, positions, share=share, seed=6400 + 10 * seed, hq=hq,
                hkv=hkv)


@pytest.mark.parametrize("seed", range(6))
def test_shared_prefix_random_geometry(cuda_device, seed):
    rng = np.random.default_rng(6500 + seed)
    hq, hkv = GROUPINGS[seed % len(GROUPINGS)]
    lp = int(rng.choice([1, 64, 130, int(rng.integers(1, 300))]))
    w = int(rng.choice([1, 64, 257, int(rng.integers(1, 600))]))
    gsize = int(rng.integers(1, 5))
    groups = int(rng.integers(1, 5))
    positions = _positions(rng, lp, w, gsize * groups, 3 * (lp + w) + 100)
    _shared_prefix_case(cuda_device, hq, hkv, lp, w, gsize, positions, seed=6600 + 10 * seed)
