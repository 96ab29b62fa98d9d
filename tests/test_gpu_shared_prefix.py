"""GPU parity of shared-prefix decode against the float64 oracle, through the C ABI.

Groups of sequences share one prompt prefix; each sequence has its own ring.  The oracle
sees, for every sequence, the plain history [0, p]: its group's prefix rows followed by its
own tokens, and attends V(p) (eq. A(i)).  The same batch also runs through plain
ps_decode_attn with the prefix copied into every sequence, so both paths are held to the
same bar: max_abs <= 2e-2, rel_rms <= 5e-3.  Rings start NaN-filled, so a read of a slot
that was never written shows up as a non-finite output.
"""
import math

import numpy as np
import pytest
import torch

import synth
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200.cache import LinearCache, PrefixSlidingCache
from tests.gpu_util import assert_close, f64
from tests.test_gpu_decode import THETA, _oracle_decode_from_history

pytestmark = pytest.mark.gpu

D = 128


def _shared_prefix_case(dev, hq, hkv, lp, w, gsize, positions, seed, scale=0.0):
    Bn = len(positions)
    assert Bn % gsize == 0
    G = Bn // gsize
    Smax = max(max(positions) + 1, lp)
    params = B.make_params(hq, hkv, D, lp, w, THETA, softmax_scale=scale)
    pre_k = synth.normal_bf16((G, lp, hkv, D), seed, dev)
    pre_v = synth.normal_bf16((G, lp, hkv, D), seed + 1, dev)
    own_k = synth.normal_bf16((Bn, Smax, hkv, D), seed + 2, dev)
    own_v = synth.normal_bf16((Bn, Smax, hkv, D), seed + 3, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), seed + 4, dev)
    # each sequence's history: its group's prefix rows, then its own tokens
    grp = torch.arange(Bn, device=dev) // gsize
    hist_k, hist_v = own_k.clone(), own_v.clone()
    hist_k[:, :lp] = pre_k[grp]
    hist_v[:, :lp] = pre_v[grp]
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    # shared store: one prefix per group (a linear cache of G sequences), rings per sequence
    shared_pre = LinearCache(G, hkv, lp, D, dev, fill=float("nan"))
    B.ps_kv_append_rope(params, shared_pre.struct, pre_k, pre_v, None,
                        torch.zeros(G, dtype=torch.int64, device=dev), lp, st)
    rings = PrefixSlidingCache(Bn, hkv, 0, w, D, dev, fill=float("nan"))
    for b, p in enumerate(positions):
        if p < lp:
            continue  # still inside the prompt: nothing in the ring yet
        view = B.make_cache(None, None, rings.k_ring[b:b + 1], rings.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, own_k[b:b + 1, lp:p + 1].contiguous(),
                            own_v[b:b + 1, lp:p + 1].contiguous(), None,
                            torch.full((1,), lp, dtype=torch.int64, device=dev), p - lp + 1, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    shared = B.make_cache(shared_pre.k, shared_pre.v, rings.k_ring, rings.v_ring, Bn)

    # the same histories in plain per-sequence stores
    plain = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    for b, p in enumerate(positions):
        view = B.make_cache(plain.k_prefix[b:b + 1], plain.v_prefix[b:b + 1],
                            plain.k_ring[b:b + 1], plain.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, hist_k[b:b + 1, :p + 1].contiguous(),
                            hist_v[b:b + 1, :p + 1].contiguous(), None,
                            torch.zeros(1, dtype=torch.int64, device=dev), p + 1, st)

    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, own_k[:, :1].contiguous(),
                        own_v[:, :1].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)

    out = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(B.ps_decode_shared_prefix_workspace_bytes(params, Bn, gsize),
                     dtype=torch.uint8, device=dev)
    B.ps_decode_attn_shared_prefix(params, shared, gsize, q, pos, out, lse, ws, st)
    out_p = torch.empty_like(out)
    lse_p = torch.empty_like(lse)
    wsp = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                      device=dev)
    B.ps_decode_attn(params, plain.struct, q, pos, out_p, lse_p, wsp, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()

    sc = scale or 1 / math.sqrt(D)
    qr, kr, vr = f64(q_raw), f64(hist_k), f64(hist_v)
    got, gl, gp, glp = f64(out), f64(lse), f64(out_p), f64(lse_p)
    for b, p in enumerate(positions):
        o, l = _oracle_decode_from_history(B_rope(qr[b], p), kr[b, :p + 1], vr[b, :p + 1], p, lp,
                                           w, sc)
        assert_close(got[b], o, f"shared b={b} p={p}")
        assert_close(gp[b], o, f"plain b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, (b, p)
        assert np.abs(glp[b] - l).max() < 2e-2, (b, p)
    return got, gp


def B_rope(q_b, p):
    import oracle as O
    return O.rope_rotate(q_b, p, THETA)


def test_shared_prefix_split_k_schedule(cuda_device):
    """15 sequences in 3 groups of 5 (30 units: the stream-K schedule, the prefix partial is
    merged as one more piece); L_prefix = 300 (a ragged third tile), W = 256; positions in
    the prompt, at the first decode token, at the cap L_prefix + W, and wrapped."""
    positions = [150, 300, 301, 555, 556, 299, 420, 700, 1000, 2047, 555, 557, 1200, 310, 999]
    _shared_prefix_case(cuda_device, 16, 2, 300, 256, 5, positions, seed=501)


def test_shared_prefix_per_unit_schedule(cuda_device):
    """160 sequences in 2 groups of 80 (320 units: one CTA per unit, the prefix partial is
    folded in at flush; 640 query rows per (group, KV head) = 5 row blocks)."""
    rng = np.random.default_rng(7)
    positions = rng.integers(130, 900, size=160).tolist()
    positions[:4] = [129, 130, 131, 193]
    _shared_prefix_case(cuda_device, 16, 2, 130, 64, 80, positions, seed=511)


def test_shared_prefix_group_seven_custom_scale(cuda_device):
    """28 query / 4 KV heads (63 rows per group and KV head), explicit softmax scale."""
    positions = [140, 200, 333, 129, 150, 1000, 64, 400, 401] * 2
    _shared_prefix_case(cuda_device, 28, 4, 130, 100, 9, positions, seed=521, scale=0.05)


def test_shared_prefix_group_size_one_equals_plain_decode(cuda_device):
    """group_size 1: every sequence owns its prefix; results match plain decode closely."""
    positions = [100, 355, 612, 999, 4000, 101]
    got, gp = _shared_prefix_case(cuda_device, 16, 2, 100, 512, 1, positions, seed=531)
    assert np.abs(got - gp).max() < 1e-2
