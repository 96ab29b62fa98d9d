"""GPU parity of the decode on seeded random geometries against the float64 oracle.

Each case draws a head grouping (1 to 8 query heads per KV head), L_prefix, W, a batch and
per-sequence positions, with positions forced onto the boundaries of eq. A(i) ("Prefix
Sliding 完全拆解", §核心机制): the last prefix row, the first window-only position, the exact
cap L_prefix + W, the first eviction, ring wrap-arounds.  Every sequence's history [0, p] is
appended through the C ABI (Continue-PE RoPE), then one decode runs, through
ps_decode_step for even cases (the step appends token p itself) and ps_decode_attn for odd
ones.  Every output row is compared with the oracle's attention over the visible set at the
floating-point bar (max_abs <= 2e-2, rel_rms <= 5e-3), and lse within 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200.cache import PrefixSlidingCache
from tests.gpu_util import assert_close, f64
from tests.test_gpu_decode import THETA, _oracle_decode_from_history, _status

pytestmark = pytest.mark.gpu

D = 128
GROUPINGS = [(16, 2), (8, 8), (28, 4), (4, 1), (7, 7), (24, 3), (8, 1), (2, 2)]


def _case(seed: int):
    """Geometry and positions of case `seed` (numpy's seeded generator; no method arithmetic)."""
    rng = np.random.default_rng(9000 + seed)
    hq, hkv = GROUPINGS[seed % len(GROUPINGS)]
    lp = int(rng.choice([0, 1, 5, 64, 100, 130, int(rng.integers(0, 300))]))
    w = int(rng.choice([1, 2, 63, 64, 65, 256, int(rng.integers(1, 700))]))
    bn = int(rng.integers(1, 13))
    edges = [lp - 1, lp, lp + 1, lp + w - 1, lp + w, lp + w + 1, lp + 2 * w, lp + 3 * w + 7]
    pos = [int(rng.integers(0, 2 * (lp + w) + 50)) for _ in range(bn)]
    for i in range(min(bn, len(edges))):
        if rng.random() < 0.6:
            pos[i] = edges[int(rng.integers(0, len(edges)))]
    pos = [max(0, p) for p in pos]
    return hq, hkv, lp, w, pos


def _run_case(dev, hq, hkv, lp, w, positions, use_step, seed):
    bn = len(positions)
    smax = max(positions) + 1
    k_raw = synth.normal_bf16((bn, smax, hkv, D), 4000 + seed, dev)
    v_raw = synth.normal_bf16((bn, smax, hkv, D), 5000 + seed, dev)
    q_raw = synth.normal_bf16((bn, hq, D), 6000 + seed, dev)
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    cache = PrefixSlidingCache(bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = _status(dev)
    # history: [0, p] for ps_decode_attn, [0, p) for ps_decode_step (it appends p itself)
    for b, p in enumerate(positions):
        n = p if use_step else p + 1
        if n == 0:
            continue
        view = B.make_cache(cache.k_prefix[b:b + 1] if lp else None,
                            cache.v_prefix[b:b + 1] if lp else None,
                            cache.k_ring[b:b + 1], cache.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, k_raw[b:b + 1, :n].contiguous(),
                            v_raw[b:b + 1, :n].contiguous(), None,
                            torch.zeros(1, dtype=torch.int64, device=dev), n, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    out = torch.full((bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((bn, hq), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, bn)), dtype=torch.uint8,
                     device=dev)
    if use_step:
        idx = torch.arange(bn, device=dev)
        k_new = k_raw[idx, pos].contiguous()
        v_new = v_raw[idx, pos].contiguous()
        B.ps_decode_step(params, cache.struct, k_new, v_new, q, pos, out, lse, ws, st)
    else:
        # q rotated at its position by a throwaway append into a scratch cache
        scratch = PrefixSlidingCache(bn, hkv, lp, w, D, dev)
        B.ps_kv_append_rope(params, scratch.struct, k_raw[:, :1].contiguous(),
                            v_raw[:, :1].contiguous(), q.view(bn, 1, hq, D), pos, 1, st)
        B.ps_decode_attn(params, cache.struct, q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    kr, vr, qr = f64(k_raw), f64(v_raw), f64(q_raw)
    got, gl = f64(out), f64(lse)
    for b, p in enumerate(positions):
        o, l = _oracle_decode_from_history(O.rope_rotate(qr[b], p, THETA), kr[b, :p + 1],
                                           vr[b, :p + 1], p, lp, w, 1 / math.sqrt(D))
        assert_close(got[b], o, f"hq={hq} hkv={hkv} lp={lp} w={w} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2


@pytest.mark.parametrize("seed", range(24))
def test_decode_random_geometry(cuda_device, seed):
    hq, hkv, lp, w, positions = _case(seed)
    _run_case(cuda_device, hq, hkv, lp, w, positions, use_step=(seed % 2 == 0), seed=seed)


def test_decode_random_per_unit_schedule(cuda_device):
    """40 sequences x 8 KV heads = 320 units, more than the 296 CTA slots: one CTA per unit,
    written straight to `out` (no split-K pieces)."""
    rng = np.random.default_rng(9100)
    lp, w = 37, 150
    positions = [int(x) for x in rng.integers(0, 500, size=40)]
    positions[:4] = [36, 37, 186, 187]
    _run_case(cuda_device, 8, 8, lp, w, positions, use_step=True, seed=100)
