"""GPU parity of the decode path (append + Continue-PE RoPE, visible ranges, split-K decode,
full-attention comparator) against the float64 oracle, through the C ABI.

Integer outputs (visible-range descriptors, ring slot of every position) must match
bit-exactly; float outputs within max_abs <= 2e-2 and rel_rms <= 5e-3.  Caches start
filled with NaN, so any read of a slot that was never written (or of an evicted key that
happens to be NaN-free) shows up as a non-finite or wrong output.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200.cache import LinearCache, PrefixSlidingCache
from tests.gpu_util import assert_close, f64

pytestmark = pytest.mark.gpu

D = 128
THETA = 1.0e6


def _status(dev):
    return torch.zeros(1, dtype=torch.int32, device=dev)


def _append_history(params, cache, k_raw, v_raw, dev, status, chunk=None):
    """Append positions 0..S-1 of every sequence (k_raw/v_raw: [B, S, Hkv, D] bf16 on dev)."""
    Bn, S = k_raw.shape[0], k_raw.shape[1]
    chunk = chunk or S
    for s0 in range(0, S, chunk):
        T = min(chunk, S - s0)
        pos0 = torch.full((Bn,), s0, dtype=torch.int64, device=dev)
        B.ps_kv_append_rope(params, cache.struct, k_raw[:, s0:s0 + T].contiguous(),
                            v_raw[:, s0:s0 + T].contiguous(), None, pos0, T, status)


# ---------------------------------------------------------------- integer checks
@pytest.mark.parametrize("lp,w", [(100, 512), (0, 7), (5, 1), (13, 64), (300, 64)])
def test_visible_ranges_bit_exact(cuda_device, lp, w):
    P = 1500
    ring = O.RingKVCache(lp, w, 1, 2, THETA)
    z = np.zeros((1, 2))
    want = {}
    probe = set(range(0, 80)) | set(range(lp + w - 3, lp + w + 3)) | {P - 1, 777, 1024}
    for p in range(P):
        ring.append(p, z, z)
        if p in probe:
            want[p] = ring.descriptor(p)
    pos = torch.tensor(sorted(want), dtype=torch.int64, device=cuda_device)
    out = torch.full((pos.numel(), 4), -7, dtype=torch.int32, device=cuda_device)
    B.ps_decode_visible_ranges(B.make_params(16, 2, D, lp, w), pos, pos.numel(), out)
    got = out.cpu().numpy()
    for i, p in enumerate(sorted(want)):
        assert tuple(got[i].tolist()) == want[p], (p, got[i], want[p])


def test_visible_ranges_large_positions(cuda_device):
    """Positions up to 2^18: closed form of the ring (pinned against the simulator on CPU)."""
    lp, w = 2000, 16384
    pos = synth.uniform_positions(257, 0, 262143, seed=5, device=cuda_device)
    out = torch.empty((257, 4), dtype=torch.int32, device=cuda_device)
    B.ps_decode_visible_ranges(B.make_params(16, 2, D, lp, w), pos, 257, out)
    got = out.cpu().numpy()
    for i, p in enumerate(pos.cpu().tolist()):
        vis = O.visible_positions(p, lp, w)
        win = vis[vis >= lp]
        slots = ((win - lp) % w).tolist()
        assert got[i, 0] == int((vis < lp).sum())
        if len(slots) == 0:
            assert tuple(got[i, 1:]) == (0, 0, 0)
            continue
        s0 = slots[0]
        l0 = min(len(slots), w - s0)
        assert slots == list(range(s0, s0 + l0)) + list(range(0, len(slots) - l0))
        assert tuple(got[i, 1:].tolist()) == (s0, l0, len(slots) - l0)


@pytest.mark.parametrize("lp,w,S,chunk", [(5, 7, 40, 40), (5, 7, 40, 3), (0, 4, 19, 19),
                                         (9, 1, 17, 5), (16, 32, 30, 30)])
def test_append_slot_map_and_rope(cuda_device, lp, w, S, chunk):
    """Every slot holds exactly the position the oracle ring says, rotated once at that
    position; slots never written stay NaN.  chunk = S appends with T > W (latest wins)."""
    Bn, hq, hkv = 3, 4, 2
    dev = cuda_device
    k_raw = synth.normal_bf16((Bn, S, hkv, D), seed=11, device=dev)
    v_raw = synth.normal_bf16((Bn, S, hkv, D), seed=12, device=dev)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    st = _status(dev)
    _append_history(params, cache, k_raw, v_raw, dev, st, chunk)
    torch.cuda.synchronize()
    assert st.item() == 0
    kr, vr = f64(k_raw), f64(v_raw)
    kp = f64(cache.k_prefix) if lp else None
    vp = f64(cache.v_prefix) if lp else None
    kg, vg = f64(cache.k_ring), f64(cache.v_ring)
    for b in range(Bn):
        ring = O.RingKVCache(lp, w, hkv, D, THETA)
        for p in range(S):
            ring.append(p, kr[b, p], vr[b, p])
        for kind, store, kt, vt, n in (("prefix", ring.prefix, kp, vp, lp),
                                       ("ring", ring.ring, kg, vg, w)):
            for idx in range(n):
                e = store[idx]
                if e is None:
                    assert np.isnan(kt[b, :, idx]).all() and np.isnan(vt[b, :, idx]).all()
                    continue
                # V copied bit-exactly: identifies which position the slot holds
                np.testing.assert_array_equal(vt[b, :, idx], e[2])
                # K rotated once at its absolute position, one bf16 rounding
                np.testing.assert_allclose(kt[b, :, idx], e[1], rtol=2 ** -7, atol=2 ** -12)


def test_append_rotates_q_in_place(cuda_device):
    dev = cuda_device
    Bn, T, hq, hkv, lp, w = 2, 5, 16, 2, 3, 4
    k = synth.normal_bf16((Bn, T, hkv, D), 21, dev)
    v = synth.normal_bf16((Bn, T, hkv, D), 22, dev)
    q = synth.normal_bf16((Bn, T, hq, D), 23, dev)
    q0 = f64(q)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    pos0 = torch.tensor([131000, 262139], dtype=torch.int64, device=dev)
    B.ps_kv_append_rope(B.make_params(hq, hkv, D, lp, w, THETA), cache.struct, k, v, q, pos0, T)
    torch.cuda.synchronize()
    got = f64(q)
    for b in range(Bn):
        for t in range(T):
            want = O.rope_rotate(q0[b, t], int(pos0[b]) + t, THETA)
            np.testing.assert_allclose(got[b, t], want, rtol=2 ** -7, atol=2 ** -11)


# ------------------------------------------------------------------ decode
def _oracle_decode_from_history(q_rot_b, kr_b, vr_b, p, lp, w, scale, theta=THETA):
    """Oracle output for one sequence whose raw history kr_b/vr_b covers [0, p]."""
    vis = O.visible_positions(p, lp, w)
    k_rot = O.rope_rotate(kr_b[vis], vis[:, None], theta)
    return O.attend_gqa(q_rot_b, k_rot, vr_b[vis], scale)


def test_decode_b1_w512_every_step(cuda_device):
    """Single-layer decode, batch 1, 16/2/128, L_prefix=100, W=512: 100-token prompt, then
    2048 decode steps (positions 100..2147); every step checked against the oracle."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_b1_w512"]
    hq, hkv, lp, w = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    steps = 2048
    S = lp + steps
    k_raw = synth.normal_bf16((1, S, hkv, D), synth.seed_for(1, 1), dev)
    v_raw = synth.normal_bf16((1, S, hkv, D), synth.seed_for(1, 2), dev)
    q_raw = synth.normal_bf16((steps, 1, hq, D), synth.seed_for(1, 3), dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    cache = PrefixSlidingCache(1, hkv, lp, w, D, dev, fill=float("nan"))
    st = _status(dev)
    pos0 = torch.zeros(1, dtype=torch.int64, device=dev)
    B.ps_kv_append_rope(params, cache.struct, k_raw[:, :lp].contiguous(),
                        v_raw[:, :lp].contiguous(), None, pos0, lp, st)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, 1)), dtype=torch.uint8, device=dev)
    outs = torch.empty((steps, 1, hq, D), dtype=torch.bfloat16, device=dev)
    lses = torch.empty((steps, 1, hq), dtype=torch.float32, device=dev)
    q = q_raw.clone()
    for i in range(steps):
        p = lp + i
        pos = torch.full((1,), p, dtype=torch.int64, device=dev)
        B.ps_kv_append_rope(params, cache.struct, k_raw[:, p:p + 1].contiguous(),
                            v_raw[:, p:p + 1].contiguous(), q[i:i + 1], pos, 1, st)
        B.ps_decode_attn(params, cache.struct, q[i], pos, outs[i], lses[i], ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    kr, vr, qr = f64(k_raw)[0], f64(v_raw)[0], f64(q_raw)
    got, got_lse = f64(outs), f64(lses)
    scale = 1 / math.sqrt(D)
    worst = 0.0
    for i in range(steps):
        p = lp + i
        qrot = O.rope_rotate(qr[i, 0], p, THETA)
        o, l = _oracle_decode_from_history(qrot, kr[:p + 1], vr[:p + 1], p, lp, w, scale)
        m, r = assert_close(got[i, 0], o, f"step {i} pos {p}")
        assert np.abs(got_lse[i, 0] - l).max() < 2e-2, f"lse step {i}"
        worst = max(worst, r)


def test_decode_b64_w4096_full_size(cuda_device):
    """Steady-state batched decode at full size (batch 64, W=4096, positions drawn in
    [8192, 131072]); three decode steps; 4 sampled sequences checked head by head."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_b64_w4096"]
    hq, hkv, lp, w, Bn = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window, wl.batch
    steps = 3
    pos_start = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, synth.seed_for(2, 0), dev)
    k_pre = synth.normal_bf16((Bn, lp, hkv, D), synth.seed_for(2, 1), dev)
    v_pre = synth.normal_bf16((Bn, lp, hkv, D), synth.seed_for(2, 2), dev)
    k_win = synth.normal_bf16((Bn, w - 1 + steps, hkv, D), synth.seed_for(2, 3), dev)
    v_win = synth.normal_bf16((Bn, w - 1 + steps, hkv, D), synth.seed_for(2, 4), dev)
    q_raw = synth.normal_bf16((steps, Bn, hq, D), synth.seed_for(2, 5), dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = _status(dev)
    B.ps_kv_append_rope(params, cache.struct, k_pre, v_pre, None,
                        torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
    # window history: positions p - W + 1 .. p - 1
    B.ps_kv_append_rope(params, cache.struct, k_win[:, :w - 1].contiguous(),
                        v_win[:, :w - 1].contiguous(), None, pos_start - (w - 1), w - 1, st)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    q = q_raw.clone()
    outs = torch.empty((steps, Bn, hq, D), dtype=torch.bfloat16, device=dev)
    lses = torch.empty((steps, Bn, hq), dtype=torch.float32, device=dev)
    for i in range(steps):
        pos = pos_start + i
        j = w - 1 + i
        B.ps_kv_append_rope(params, cache.struct, k_win[:, j:j + 1].contiguous(),
                            v_win[:, j:j + 1].contiguous(), q[i], pos, 1, st)
        B.ps_decode_attn(params, cache.struct, q[i], pos, outs[i], lses[i], ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    scale = 1 / math.sqrt(D)
    P = pos_start.cpu().numpy()
    kp, vp, kw, vw, qr = f64(k_pre), f64(v_pre), f64(k_win), f64(v_win), f64(q_raw)
    got, got_lse = f64(outs), f64(lses)
    for b in (0, 17, 40, 63):
        for i in range(steps):
            p = int(P[b]) + i
            vis = O.visible_positions(p, lp, w)
            assert len(vis) == lp + w
            base = int(P[b]) - (w - 1)  # position of k_win[:, 0]
            kr = np.stack([kp[b, x] if x < lp else kw[b, x - base] for x in vis])
            vr = np.stack([vp[b, x] if x < lp else vw[b, x - base] for x in vis])
            k_rot = O.rope_rotate(kr, vis[:, None], THETA)
            o, l = O.attend_gqa(O.rope_rotate(qr[i, b], p, THETA), k_rot, vr, scale)
            assert_close(got[i, b], o, f"b={b} step={i}")
            assert np.abs(got_lse[i, b] - l).max() < 2e-2


@pytest.mark.parametrize("Bn", [32, 128])
def test_decode_equal_lengths_unit_aligned_waves(cuda_device, Bn):
    """Batch 32 and 128 at W=4096 with every sequence past L_prefix + W: the stream-K wave is
    then a multiple of the unit count (64 units x 4 CTAs, 256 units x 2), so each CTA streams
    a whole part of one unit and the merge combines exactly that many pieces.  One decode
    step through ps_decode_step; 5 sampled sequences checked head by head."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_b64_w4096"]
    hq, hkv, lp, w = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    seed = lambda k: synth.seed_for(20 + Bn, k)  # noqa: E731
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, seed(0), dev)
    k_pre = synth.normal_bf16((Bn, lp, hkv, D), seed(1), dev)
    v_pre = synth.normal_bf16((Bn, lp, hkv, D), seed(2), dev)
    k_win = synth.normal_bf16((Bn, w, hkv, D), seed(3), dev)
    v_win = synth.normal_bf16((Bn, w, hkv, D), seed(4), dev)
    q_raw = synth.normal_bf16((Bn, hq, D), seed(5), dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = _status(dev)
    B.ps_kv_append_rope(params, cache.struct, k_pre, v_pre, None,
                        torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
    # window history: positions p - W + 1 .. p - 1; the step appends position p itself
    B.ps_kv_append_rope(params, cache.struct, k_win[:, :w - 1].contiguous(),
                        v_win[:, :w - 1].contiguous(), None, pos - (w - 1), w - 1, st)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    q = q_raw.clone()
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Bn, hq), dtype=torch.float32, device=dev)
    B.ps_decode_step(params, cache.struct, k_win[:, w - 1].contiguous(),
                     v_win[:, w - 1].contiguous(), q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    scale = 1 / math.sqrt(D)
    P = pos.cpu().numpy()
    kp, vp, kw, vw, qr = f64(k_pre), f64(v_pre), f64(k_win), f64(v_win), f64(q_raw)
    got, got_lse = f64(out), f64(lse)
    for b in (0, 1, Bn // 2, Bn - 2, Bn - 1):
        p = int(P[b])
        vis = O.visible_positions(p, lp, w)
        assert len(vis) == lp + w
        base = p - (w - 1)  # position of k_win[:, 0]
        kr = np.stack([kp[b, x] if x < lp else kw[b, x - base] for x in vis])
        vr = np.stack([vp[b, x] if x < lp else vw[b, x - base] for x in vis])
        k_rot = O.rope_rotate(kr, vis[:, None], THETA)
        o, l = O.attend_gqa(O.rope_rotate(qr[b], p, THETA), k_rot, vr, scale)
        assert_close(got[b], o, f"Bn={Bn} b={b}")
        assert np.abs(got_lse[b] - l).max() < 2e-2


@pytest.mark.parametrize("lp,w,positions", [
    (0, 64, [0, 1, 63, 64, 65, 200]),            # pure sliding window
    (7, 1, [0, 6, 7, 8, 50]),                     # window of one
    (50, 30, [10, 49, 50, 79, 80, 81, 159, 300]),  # warm-up, exact cap, wraps
    (130, 64, [129, 130, 193, 194, 257, 401]),    # prefix longer than two tiles
    (3, 200, [2, 202, 203, 204, 403, 404, 405]),  # wrap at the ring end
])
def test_decode_edge_cases_mixed_batch(cuda_device, lp, w, positions):
    """Mixed positions in one batch (warm-up, exact cap L_prefix+W, ring wrap, W=1,
    L_prefix=0), with history appended in one call (T > W: latest wins)."""
    dev = cuda_device
    hq, hkv = 16, 2
    Bn = len(positions)
    Smax = max(positions) + 1
    k_raw = synth.normal_bf16((Bn, Smax, hkv, D), 31, dev)
    v_raw = synth.normal_bf16((Bn, Smax, hkv, D), 32, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), 33, dev)
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = _status(dev)
    # per-sequence history [0, p]: append into a batch-1 view of each sequence
    for b, p in enumerate(positions):
        view = B.make_cache(cache.k_prefix[b:b + 1] if lp else None,
                            cache.v_prefix[b:b + 1] if lp else None,
                            cache.k_ring[b:b + 1], cache.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, k_raw[b:b + 1, :p + 1].contiguous(),
                            v_raw[b:b + 1, :p + 1].contiguous(), None,
                            torch.zeros(1, dtype=torch.int64, device=dev), p + 1, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    # rotate q at its position with a throwaway append into a scratch cache
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, k_raw[:, :1].contiguous(),
                        v_raw[:, :1].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Bn, hq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    B.ps_decode_attn(params, cache.struct, q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    kr, vr, qr = f64(k_raw), f64(v_raw), f64(q_raw)
    got, gl = f64(out), f64(lse)
    for b, p in enumerate(positions):
        o, l = _oracle_decode_from_history(O.rope_rotate(qr[b], p, THETA), kr[b, :p + 1],
                                           vr[b, :p + 1], p, lp, w, 1 / math.sqrt(D))
        assert_close(got[b], o, f"lp={lp} w={w} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2


def test_decode_group_seven_and_custom_scale(cuda_device):
    """7B-class grouping (28 query / 4 KV heads) and an explicit softmax scale."""
    dev = cuda_device
    hq, hkv, lp, w, p = 28, 4, 20, 100, 333
    k_raw = synth.normal_bf16((1, p + 1, hkv, D), 41, dev)
    v_raw = synth.normal_bf16((1, p + 1, hkv, D), 42, dev)
    q_raw = synth.normal_bf16((1, hq, D), 43, dev)
    params = B.make_params(hq, hkv, D, lp, w, THETA, softmax_scale=0.05)
    cache = PrefixSlidingCache(1, hkv, lp, w, D, dev, fill=float("nan"))
    B.ps_kv_append_rope(params, cache.struct, k_raw, v_raw, None,
                        torch.zeros(1, dtype=torch.int64, device=dev), p + 1)
    q = q_raw.clone()
    pos = torch.tensor([p], dtype=torch.int64, device=dev)
    scratch = PrefixSlidingCache(1, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, k_raw[:, :1].contiguous(),
                        v_raw[:, :1].contiguous(), q.view(1, 1, hq, D), pos, 1)
    out = torch.empty((1, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, 1)), dtype=torch.uint8, device=dev)
    B.ps_decode_attn(params, cache.struct, q, pos, out, None, ws)
    torch.cuda.synchronize()
    o, _ = _oracle_decode_from_history(O.rope_rotate(f64(q_raw)[0], p, THETA), f64(k_raw)[0],
                                       f64(v_raw)[0], p, lp, w, 0.05)
    assert_close(f64(out)[0], o, "group 7")


def test_decode_bad_position_sets_status_and_zeroes(cuda_device):
    dev = cuda_device
    hq, hkv, lp, w = 16, 2, 4, 8
    cache = PrefixSlidingCache(2, hkv, lp, w, D, dev)
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    q = synth.normal_bf16((2, hq, D), 51, dev)
    pos = torch.tensor([-3, 5], dtype=torch.int64, device=dev)
    out = torch.full((2, hq, D), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.zeros((2, hq), dtype=torch.float32, device=dev)
    st = _status(dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, 2)), dtype=torch.uint8, device=dev)
    B.ps_decode_attn(params, cache.struct, q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() & B.PS_DEV_BAD_POS
    assert (out[0] == 0).all() and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    assert torch.isfinite(out[1].float()).all()


# ------------------------------------------------------------ full attention
@pytest.mark.parametrize("positions,lmax", [([0, 5, 127, 128, 1000], 1001), ([63, 64, 65], 300)])
def test_full_attention_comparator(cuda_device, positions, lmax):
    dev = cuda_device
    hq, hkv = 16, 2
    Bn = len(positions)
    k_raw = synth.normal_bf16((Bn, lmax, hkv, D), 61, dev)
    v_raw = synth.normal_bf16((Bn, lmax, hkv, D), 62, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), 63, dev)
    lin = LinearCache(Bn, hkv, lmax, D, dev, fill=float("nan"))
    lp_params = lin.params(hq, THETA)
    st = _status(dev)
    # fill positions [0, p] of each sequence only; the rest stays NaN
    for b, p in enumerate(positions):
        view = B.make_cache(lin.k[b:b + 1], lin.v[b:b + 1], None, None, 1)
        B.ps_kv_append_rope(lp_params, view, k_raw[b:b + 1, :p + 1].contiguous(),
                            v_raw[b:b + 1, :p + 1].contiguous(), None,
                            torch.zeros(1, dtype=torch.int64, device=dev), p + 1, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    scratch = LinearCache(Bn, hkv, lmax, D, dev)
    B.ps_kv_append_rope(lp_params, scratch.struct, k_raw[:, :1].contiguous(),
                        v_raw[:, :1].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    params = B.make_params(hq, hkv, D, 0, 1, THETA)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Bn, hq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_full_attn_workspace_bytes(params, Bn, lmax)), dtype=torch.uint8,
                     device=dev)
    B.ps_full_attn_ref(params, lin.k, lin.v, lmax, q, pos, Bn, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    kr, vr, qr = f64(k_raw), f64(v_raw), f64(q_raw)
    for b, p in enumerate(positions):
        k_rot = O.rope_rotate(kr[b, :p + 1], np.arange(p + 1)[:, None], THETA)
        o, l = O.full_attention_decode(O.rope_rotate(qr[b], p, THETA), k_rot, vr[b], p,
                                       1 / math.sqrt(D))
        assert_close(f64(out)[b], o, f"full p={p}")
        assert np.abs(f64(lse)[b] - l).max() < 2e-2


def test_full_attention_position_out_of_range(cuda_device):
    dev = cuda_device
    lin = LinearCache(1, 2, 64, D, dev)
    params = B.make_params(16, 2, D, 0, 1, THETA)
    q = synth.normal_bf16((1, 16, D), 71, dev)
    out = torch.empty((1, 16, D), dtype=torch.bfloat16, device=dev)
    st = _status(dev)
    ws = torch.empty(max(1, B.ps_full_attn_workspace_bytes(params, 1, 64)), dtype=torch.uint8,
                     device=dev)
    B.ps_full_attn_ref(params, lin.k, lin.v, 64, q, torch.tensor([64], device=dev), 1, out, None,
                       ws, st)
    torch.cuda.synchronize()
    assert st.item() & B.PS_DEV_POS_RANGE
    assert (out == 0).all()


def test_prefix_sliding_equals_full_attention_in_warmup(cuda_device):
    """n <= L_prefix + W: the PS decode and the full-attention kernel agree (warm-up)."""
    dev = cuda_device
    hq, hkv, lp, w = 16, 2, 40, 100
    p = lp + w - 1
    k_raw = synth.normal_bf16((1, p + 1, hkv, D), 81, dev)
    v_raw = synth.normal_bf16((1, p + 1, hkv, D), 82, dev)
    q = synth.normal_bf16((1, hq, D), 83, dev)
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    cache = PrefixSlidingCache(1, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, cache.struct, k_raw, v_raw, None,
                        torch.zeros(1, dtype=torch.int64, device=dev), p + 1)
    lin = LinearCache(1, hkv, p + 1, D, dev)
    B.ps_kv_append_rope(lin.params(hq, THETA), lin.struct, k_raw, v_raw, None,
                        torch.zeros(1, dtype=torch.int64, device=dev), p + 1)
    pos = torch.tensor([p], dtype=torch.int64, device=dev)
    o1 = torch.empty((1, hq, D), dtype=torch.bfloat16, device=dev)
    o2 = torch.empty_like(o1)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=dev)
    B.ps_decode_attn(params, cache.struct, q, pos, o1, None, ws)
    B.ps_full_attn_ref(B.make_params(hq, hkv, D, 0, 1), lin.k, lin.v, p + 1, q, pos, 1, o2, None,
                       ws)
    torch.cuda.synchronize()
    assert_close(f64(o1), f64(o2), "warm-up PS vs full")


@pytest.mark.parametrize("Bn,lp,w,lo,hi", [(64, 100, 4096, 8192, 131072),   # stream-K
                                         (160, 100, 256, 0, 4000),         # one CTA per unit
                                         (5, 300, 64, 0, 400),             # prompt / warm-up
                                         (40, 100, 4096, 0, 131072)])      # mixed lengths
def test_decode_step_equals_append_then_decode(cuda_device, Bn, lp, w, lo, hi):
    """ps_decode_step (the decode streams before the append finishes, except the newest row)
    is bit-identical to ps_kv_append_rope followed by ps_decode_attn: the rotated query,
    outputs, lse, status and every row of the cache.  The mixed batch puts short sequences
    (one or two tiles, each inside one CTA's share) next to long ones (about seven stream-K
    pieces each, two rounds of the merge's four-piece combine)."""
    dev = cuda_device
    hq, hkv = 16, 2
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    pos = synth.uniform_positions(Bn, lo, hi, seed=77, device=dev)
    if Bn == 5:
        pos[0] = -3  # a bad position: both paths flag it and write zeros
    if Bn == 40:
        short = synth.uniform_positions(Bn, 0, 100, seed=76, device=dev)
        pos[0::2] = short[0::2]
        pos[1::2] = pos[1::2].clamp(min=65536)
    caches = []
    for _ in range(2):
        c = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
        if lp:
            c.k_prefix.copy_(synth.normal_bf16(c.k_prefix.shape, 78, dev))
            c.v_prefix.copy_(synth.normal_bf16(c.v_prefix.shape, 79, dev))
        c.k_ring.copy_(synth.normal_bf16(c.k_ring.shape, 80, dev))
        c.v_ring.copy_(synth.normal_bf16(c.v_ring.shape, 81, dev))
        caches.append(c)
    k_new = synth.normal_bf16((Bn, 1, hkv, D), 82, dev)
    v_new = synth.normal_bf16((Bn, 1, hkv, D), 83, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), 84, dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8, device=dev)
    outs = []
    for i, c in enumerate(caches):
        q = q_raw.clone()
        out = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        if i == 0:
            B.ps_kv_append_rope(params, c.struct, k_new, v_new, q.view(Bn, 1, hq, D), pos, 1, st)
            B.ps_decode_attn(params, c.struct, q, pos, out, lse, ws, st)
        else:
            B.ps_decode_step(params, c.struct, k_new, v_new, q, pos, out, lse, ws, st)
        torch.cuda.synchronize()
        outs.append((q, out, lse, st.item()))
    (qa, oa, la, sa), (qb, ob, lb, sb) = outs
    assert sa == sb
    assert torch.equal(qa, qb) and torch.equal(oa, ob) and torch.equal(la, lb)
    for a, b in ((caches[0].k_ring, caches[1].k_ring), (caches[0].v_ring, caches[1].v_ring)):
        assert torch.equal(a, b)
    if lp:
        assert torch.equal(caches[0].k_prefix, caches[1].k_prefix)
        assert torch.equal(caches[0].v_prefix, caches[1].v_prefix)


def test_graph_launched_steps_equal_eager_steps(cuda_device):
    """The launch configuration bench.py times: ps_decode_step on the batch-64, W=4096
    workload replayed as one CUDA graph of 8 steps is bit-identical (q, out, cache) to the
    same 8 steps launched one by one."""
    import bench
    dev = cuda_device
    wl = synth.WORKLOADS["decode_b64_w4096"]
    K = 8
    runs = []
    for graph in (False, True):
        work = bench.DecodeWorkload(wl, dev, 0, K)
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(K):
                    work.step(i)
            g.replay()
        else:
            for i in range(K):
                work.step(i)
        torch.cuda.synchronize()
        assert work.status.item() == 0
        runs.append((work.q.clone(), work.out.clone(), work.cache.k_ring.clone(),
                     work.cache.v_ring.clone()))
        del work
        torch.cuda.empty_cache()
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    assert torch.isfinite(runs[1][1].float()).all()
