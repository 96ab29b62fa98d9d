"""GPU parity of the masked prefill (forward and backward) on seeded random geometries.

Each case draws a sequence length, L_prefix, W and a head grouping (with L_prefix and W
often on tile boundaries or past the sequence), then checks, against the float64 oracle
("Prefix Sliding 完全拆解", §核心机制 eq. A(i) for the mask, §Kernel 实现 for the tile plan):
the tile plan bit-exact, every output row and lse of the forward (max_abs <= 2e-2,
rel_rms <= 5e-3), and for every other case every row of dQ and key of dK, dV of the
backward (the bar of tests/test_gpu_prefill_bwd.py, derived from the kernels' rounding
model).
"""
import math

import numpy as np
import pytest

import oracle as O
from tests.test_gpu_prefill import _check_rows, _run
from tests.test_gpu_prefill_bwd import _check_all, _forward_backward

pytestmark = pytest.mark.gpu

D = 128
GROUPINGS = [(4, 2), (8, 1), (7, 7), (6, 3), (28, 4), (2, 2)]


def _case(seed: int):
    """Geometry of case `seed` (numpy's seeded generator; no method arithmetic)."""
    rng = np.random.default_rng(7000 + seed)
    hq, hkv = GROUPINGS[seed % len(GROUPINGS)]
    s = int(rng.choice([1, 127, 128, 129, 255, 256, int(rng.integers(2, 700))]))
    lp = int(rng.choice([0, 1, 127, 128, 129, s, s + 5, int(rng.integers(0, s + 1))]))
    w = int(rng.choice([1, 2, 127, 128, 129, 256, s, int(rng.integers(1, 900))]))
    return s, lp, w, hq, hkv


@pytest.mark.parametrize("seed", range(12))
def test_prefill_random_geometry(cuda_device, seed):
    s, lp, w, hq, hkv = _case(seed)
    q, k, v, out, lse, plan = _run(cuda_device, 2, s, hq, hkv, lp, w, seed=800 + seed)
    np.testing.assert_array_equal(plan.cpu().numpy(), O.tile_plan(s, lp, w, 128, 128))
    _check_rows(q, k, v, out, lse, lp, w, list(range(s)))


@pytest.mark.parametrize("seed", range(0, 12, 2))
def test_prefill_bwd_random_geometry(cuda_device, seed):
    s, lp, w, hq, hkv = _case(seed)
    _, inputs, grads, _ = _forward_backward(cuda_device, 1, s, hq, hkv, lp, w, seed=900 + seed)
    _check_all(inputs, grads, lp, w, 1 / math.sqrt(D))
