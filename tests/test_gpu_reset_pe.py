"""GPU parity of Reset-PE decode against the float64 oracle, through the C ABI.

The oracle applies Reset PE literally ("Prefix Sliding 完全拆解", §位置编码): the window is
renumbered to follow the prefix and every visible key and the query are rotated at those
ids.  The library decodes from the ordinary Continue-PE cache and rotates only the query
again for the prefix rows.  A second, literal path is checked too: the window re-appended
at its renumbered ids into a fresh cache, then plain decode at the query's id.
Bar: max_abs <= 2e-2, rel_rms <= 5e-3; lse within 2e-2.
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

pytestmark = pytest.mark.gpu

D = 128
THETA = 1.0e6


def _setup(dev, hq, hkv, lp, w, positions, seed, scale=0.0):
    Bn = len(positions)
    Smax = max(positions) + 1
    params = B.make_params(hq, hkv, D, lp, w, THETA, softmax_scale=scale)
    k_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed, dev)
    v_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed + 1, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), seed + 2, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    for b, p in enumerate(positions):
        # only the visible history matters; append [0, p] in one call (latest wins)
        view = B.make_cache(cache.k_prefix[b:b + 1] if lp else None,
                            cache.v_prefix[b:b + 1] if lp else None,
                            cache.k_ring[b:b + 1], cache.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, k_raw[b:b + 1, :p + 1].contiguous(),
                            v_raw[b:b + 1, :p + 1].contiguous(), None,
                            torch.zeros(1, dtype=torch.int64, device=dev), p + 1, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, k_raw[:, :1].contiguous(),
                        v_raw[:, :1].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return params, cache, pos, q, (q_raw, k_raw, v_raw), st


def _decode(fn, params, cache, q, pos, st):
    Bn, hq = q.shape[0], q.shape[1]
    out = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=q.device)
    lse = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=q.device)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=q.device)
    fn(params, cache.struct, q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return out, lse


def _check_oracle(out, lse, raw, positions, lp, w, scale, what):
    qr, kr, vr = (f64(t) for t in raw)
    got, gl = f64(out), f64(lse)
    for b, p in enumerate(positions):
        o, l = O.reset_pe_decode_reference(qr[b], kr[b, :p + 1], vr[b, :p + 1], p, lp, w, THETA,
                                           scale)
        assert_close(got[b], o, f"{what} b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, (what, b, p)


@pytest.mark.parametrize("lp,w,positions", [
    (100, 512, [99, 100, 611, 612, 613, 1000, 2047, 5000]),   # warm-up, cap, evicted
    (130, 64, [129, 193, 194, 300, 777, 1500]),               # prefix longer than two tiles
    (7, 1, [6, 7, 8, 50]),                                    # window of one
])
def test_reset_pe_decode_matches_oracle(cuda_device, lp, w, positions):
    params, cache, pos, q, raw, st = _setup(cuda_device, 16, 2, lp, w, positions, seed=601)
    out, lse = _decode(B.ps_decode_attn_reset_pe, params, cache, q, pos, st)
    _check_oracle(out, lse, raw, positions, lp, w, 1 / math.sqrt(D), "reset")


def test_reset_pe_per_unit_schedule_and_large_positions(cuda_device):
    """160 sequences (one CTA per unit) at positions up to 2^17: the extra query rotation
    spans ~1.3e5 ids, reduced modulo 2 pi in float64."""
    rng = np.random.default_rng(11)
    positions = rng.integers(3000, 131072, size=160).tolist()
    lp, w = 100, 256
    params, cache, pos, q, raw, st = _setup(cuda_device, 16, 2, lp, w, positions, seed=611)
    out, lse = _decode(B.ps_decode_attn_reset_pe, params, cache, q, pos, st)
    idx = list(range(0, 160, 9))
    _check_oracle(out[idx], lse[idx], tuple(t[idx] for t in raw), [positions[i] for i in idx],
                  lp, w, 1 / math.sqrt(D), "reset per-unit")


def test_reset_pe_equals_continue_pe_when_ids_do_not_move(cuda_device):
    """Warm-up (nothing evicted) and L_prefix = 0: the extra rotation is by 0, so the
    result is bit-identical to ps_decode_attn."""
    for lp, w, positions in [(100, 512, [100, 300, 611]), (0, 64, [10, 63, 64, 500])]:
        params, cache, pos, q, raw, st = _setup(cuda_device, 16, 2, lp, w, positions, seed=621)
        a, la = _decode(B.ps_decode_attn_reset_pe, params, cache, q, pos, st)
        b, lb = _decode(B.ps_decode_attn, params, cache, q, pos, st)
        assert torch.equal(a, b) and torch.equal(la, lb)


def test_reset_pe_group_seven_custom_scale(cuda_device):
    positions = [20, 119, 120, 121, 333, 4000]
    params, cache, pos, q, raw, st = _setup(cuda_device, 28, 4, 20, 100, positions, seed=631,
                                            scale=0.05)
    out, lse = _decode(B.ps_decode_attn_reset_pe, params, cache, q, pos, st)
    _check_oracle(out, lse, raw, positions, 20, 100, 0.05, "reset group 7")


def test_reset_pe_literal_recompute_path(cuda_device):
    """The literal way: re-append the visible window at its Reset-PE ids (L_prefix, ...) into
    a fresh cache and decode at the query's id.  Same oracle, same bar."""
    dev = cuda_device
    lp, w, hq, hkv = 100, 512, 16, 2
    positions = [700, 1000, 4000, 612]
    params, cache, pos, q, raw, st = _setup(dev, hq, hkv, lp, w, positions, seed=641)
    q_raw, k_raw, v_raw = raw
    fresh = PrefixSlidingCache(len(positions), hkv, lp, w, D, dev, fill=float("nan"))
    q2 = q_raw.clone()
    qid = []
    for b, p in enumerate(positions):
        vis, ids, q_id = O.reset_pe_positions(p, lp, w)
        qid.append(q_id)
        view = B.make_cache(fresh.k_prefix[b:b + 1], fresh.v_prefix[b:b + 1],
                            fresh.k_ring[b:b + 1], fresh.v_ring[b:b + 1], 1)
        sel = torch.tensor(vis, device=dev)
        T = len(vis)
        # prefix rows keep their ids; window rows land at ids L_prefix .. q_id
        q_rows = torch.zeros((1, T, hq, D), dtype=torch.bfloat16, device=dev)
        q_rows[0, -1] = q_raw[b]
        B.ps_kv_append_rope(params, view, k_raw[b:b + 1, sel].contiguous(),
                            v_raw[b:b + 1, sel].contiguous(), q_rows,
                            torch.zeros(1, dtype=torch.int64, device=dev), T, st)
        q2[b] = q_rows[0, -1]
    qpos = torch.tensor(qid, dtype=torch.int64, device=dev)
    out, lse = _decode(B.ps_decode_attn, params, fresh, q2, qpos, st)
    _check_oracle(out, lse, raw, positions, lp, w, 1 / math.sqrt(D), "literal")
