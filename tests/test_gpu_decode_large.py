"""GPU parity of the decode path at the long-trace and full-stack geometries, through the C ABI.

The sweep workload (batch 256, 16/2/128, L_prefix 100, W 8192, positions 4K .. 128K) and one
layer of the full-stack workload (batch 1024, L_prefix 2000, W 16384, positions up to 2^18)
have more (sequence, KV head) units than the GPU has CTA slots, so the decode runs its
one-CTA-per-unit schedule there, not the stream-K one the batch-64 workload uses.  These
tests run those exact launches and check sampled sequences head by head against the float64
oracle ("Prefix Sliding 完全拆解", §核心机制, eq. A(i) and eq. L_total): every key the query
may see, and no other, with RoPE at absolute positions (§位置编码, Continue PE).

The full-attention comparator is checked the same way at 131K positions, on both schedules.
Finally, decode at position p (ps_decode_step) is cross-checked against row p of the masked
prefill over the same rotated sequence (the warm-up paragraph of §核心机制: the same mask
whether a row is produced by decode or by prefill).

Caches start NaN-filled wherever the test writes nothing, so a read of a row outside the
visible set shows up as a non-finite or wrong output.
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


def _view(cache, b0, b1):
    """The cache of sequences [b0, b1) (a contiguous slice along the batch axis)."""
    lp = cache.k_prefix is not None
    return B.make_cache(cache.k_prefix[b0:b1] if lp else None,
                        cache.v_prefix[b0:b1] if lp else None,
                        cache.k_ring[b0:b1], cache.v_ring[b0:b1], b1 - b0)


def _runs(values):
    """[(start, end, value)] for the maximal runs of equal values."""
    out, s = [], 0
    for i in range(1, len(values) + 1):
        if i == len(values) or values[i] != values[s]:
            out.append((s, i, values[s]))
            s = i
    return out


def _fill_history(params, cache, pos, lp, w, hkv, sample, seed, dev, st, chunk=2048):
    """Appends every sequence's visible history except its own position P_b: prefix rows
    [0, L_prefix) and window positions [max(L_prefix, P_b - W + 1), P_b), raw N(0,1) keys
    and values rotated by the append kernel.  Every P_b >= L_prefix; sequences with the same
    window length must be contiguous in the batch.  Returns, for each sampled sequence, the
    positions it was given and their raw keys and values (host bf16, position order)."""
    P = [int(x) for x in pos.cpu().tolist()]
    Bn = len(P)
    assert min(P) >= lp
    parts = {b: [] for b in sample}

    def keep(kk, vv, b0, starts):
        rows = [b for b in sample if b0 <= b < b0 + kk.shape[0]]
        if not rows:
            return
        sel = torch.tensor([b - b0 for b in rows], device=kk.device)
        kc, vc = kk[sel].cpu(), vv[sel].cpu()
        for r, b in enumerate(rows):
            parts[b].append((starts[b - b0], kc[r], vc[r]))

    if lp:
        k = synth.normal_bf16((Bn, lp, hkv, D), seed, dev)
        v = synth.normal_bf16((Bn, lp, hkv, D), seed + 1, dev)
        B.ps_kv_append_rope(params, cache.struct, k, v, None,
                            torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
        keep(k, v, 0, [0] * Bn)
    lens = [min(w - 1, p - lp) for p in P]
    for b0, b1, L in _runs(lens):
        if L == 0:
            continue
        view = _view(cache, b0, b1)
        start = [max(lp, P[b] - w + 1) for b in range(b0, b1)]
        start_t = torch.tensor(start, dtype=torch.int64, device=dev)
        for c0 in range(0, L, chunk):
            T = min(chunk, L - c0)
            k = synth.normal_bf16((b1 - b0, T, hkv, D), seed + 2 + 7 * b0 + 131 * c0, dev)
            v = synth.normal_bf16((b1 - b0, T, hkv, D), seed + 3 + 7 * b0 + 131 * c0, dev)
            B.ps_kv_append_rope(params, view, k, v, None, start_t + c0, T, st)
            keep(k, v, b0, [s + c0 for s in start])
    raw = {}
    for b, chunks in parts.items():
        chunks.sort(key=lambda c: c[0])
        positions = np.concatenate([np.arange(s, s + kc.shape[0]) for s, kc, _ in chunks])
        raw[b] = (positions, torch.cat([kc for _, kc, _ in chunks]),
                  torch.cat([vc for _, _, vc in chunks]))
    return raw


def _step_and_check(params, cache, pos, lp, w, hq, hkv, raw, seed, dev, st):
    """Appends the new token at pos and decodes it twice: ps_kv_append_rope + ps_decode_attn
    on one copy of the cache, ps_decode_step on another.  Rotated queries, outputs, lse and
    caches must be bit-identical.  Sampled sequences are checked against the oracle on every
    head and the lse."""
    Bn = pos.numel()
    k_new = synth.normal_bf16((Bn, 1, hkv, D), seed, dev)
    v_new = synth.normal_bf16((Bn, 1, hkv, D), seed + 1, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), seed + 2, dev)
    nb = B.ps_decode_workspace_bytes(params, Bn)
    ws = torch.empty(max(1, nb), dtype=torch.uint8, device=dev)
    twin = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
    for a, b in ((twin.k_prefix, cache.k_prefix), (twin.v_prefix, cache.v_prefix),
                 (twin.k_ring, cache.k_ring), (twin.v_ring, cache.v_ring)):
        a.copy_(b)
    q1 = q_raw.clone()
    out1 = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse1 = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
    B.ps_kv_append_rope(params, cache.struct, k_new, v_new, q1.view(Bn, 1, hq, D), pos, 1, st)
    B.ps_decode_attn(params, cache.struct, q1, pos, out1, lse1, ws, st)
    q2 = q_raw.clone()
    out2 = torch.full_like(out1, float("nan"))
    lse2 = torch.full_like(lse1, float("nan"))
    B.ps_decode_step(params, twin.struct, k_new.view(Bn, hkv, D), v_new.view(Bn, hkv, D), q2,
                     pos, out2, lse2, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2) and torch.equal(q1, q2)
    for a, b in ((twin.k_prefix, cache.k_prefix), (twin.v_prefix, cache.v_prefix),
                 (twin.k_ring, cache.k_ring), (twin.v_ring, cache.v_ring)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))  # bits, NaN canaries too
    del twin
    P = pos.cpu().tolist()
    kn, vn, qr = f64(k_new), f64(v_new), f64(q_raw)
    got, gl = f64(out1), f64(lse1)
    scale = 1 / math.sqrt(D)
    for b, (hist, kh, vh) in raw.items():
        p = int(P[b])
        vis = O.visible_positions(p, lp, w)
        assert len(vis) == min(p + 1, lp + w)
        assert hist.tolist() + [p] == vis.tolist(), f"history of sequence {b} is not V(p) - {{p}}"
        kr = np.concatenate([kh.double().numpy(), kn[b]], axis=0)
        vr = np.concatenate([vh.double().numpy(), vn[b]], axis=0)
        k_rot = O.rope_rotate(kr, vis[:, None], THETA)
        o, l = O.attend_gqa(O.rope_rotate(qr[b], p, THETA), k_rot, vr, scale)
        assert_close(got[b], o, f"b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, f"lse b={b} p={p}"
    assert torch.isfinite(out1.float()).all()


def test_decode_sweep_geometry_per_unit_schedule(cuda_device):
    """Batch 256, 16/2/128, L_prefix 100, W 8192; sequences at the sweep's positions
    4K, 8K (both still in warm-up: n <= L_prefix + W), 16K, 32K, 64K and 128K (full
    windows, each with its own wrap point).  512 units: one CTA per unit."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_sweep_b256_w8192"]
    Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    assert B.ps_decode_workspace_bytes(params, Bn) == 0  # per-unit schedule: no partials
    points = (4096, 8192, 16384, 32768, 65536, 131072)
    g = torch.Generator().manual_seed(synth.seed_for(wl.index, 20))
    jitter = torch.randint(0, 8192, (Bn,), generator=g).tolist()
    cls = [i * len(points) // Bn for i in range(Bn)]  # contiguous classes
    P = [points[c] + (jitter[i] if points[c] > lp + w else 0) for i, c in enumerate(cls)]
    pos = torch.tensor(P, dtype=torch.int64, device=dev)
    sample = sorted({b for c in range(len(points)) for b in
                     (cls.index(c), len(cls) - 1 - cls[::-1].index(c))})
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    raw = _fill_history(params, cache, pos, lp, w, hkv, sample, synth.seed_for(wl.index, 21),
                        dev, st)
    _step_and_check(params, cache, pos, lp, w, hq, hkv, raw, synth.seed_for(wl.index, 22), dev,
                    st)


def test_decode_full_stack_layer_geometry(cuda_device):
    """One layer of the full-stack workload: batch 1024, 16/2/128, L_prefix 2000, W 16384,
    positions drawn in [32768, 262143] (angles up to 2^18 rad * theta^0).  2048 units: one
    CTA per unit, 18,384 visible keys each."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_stack_l28_b1024_w16384"]
    Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    assert B.ps_decode_workspace_bytes(params, Bn) == 0
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi - 1, synth.seed_for(wl.index, 20), dev)
    P = pos.cpu()
    sample = sorted({int(P.argmin()), int(P.argmax()), 0, 1, 511, 700, 1022, 1023})
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    raw = _fill_history(params, cache, pos, lp, w, hkv, sample, synth.seed_for(wl.index, 21),
                        dev, st, chunk=1024)
    _step_and_check(params, cache, pos, lp, w, hq, hkv, raw, synth.seed_for(wl.index, 22), dev,
                    st)


@pytest.mark.parametrize("Bn,points", [
    (64, None),                                            # batch-64 positions: stream-K
    (256, (4096, 8192, 16384, 32768, 65536, 131072)),      # sweep positions: one CTA per unit
])
def test_full_attention_long_positions(cuda_device, Bn, points):
    """ps_full_attn_ref over a linear cache of 131K+ positions.  Every key in [0, p] is
    attended; rows past p stay NaN."""
    dev = cuda_device
    hq, hkv = 16, 2
    if points is None:
        wl = synth.WORKLOADS["decode_b64_w4096"]
        pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, synth.seed_for(wl.index, 30), dev)
        pos[0] = wl.pos_hi  # the longest history of the workload
    else:
        P = [points[i * len(points) // Bn] + i % 5 for i in range(Bn)]
        pos = torch.tensor(P, dtype=torch.int64, device=dev)
    P = pos.cpu().tolist()
    lmax = max(P) + 1
    assert lmax >= 131073
    sample = sorted({0, int(np.argmax(P)), int(np.argmin(P)), Bn // 2, Bn - 1})
    lin = LinearCache(Bn, hkv, lmax, D, dev, fill=None)
    aparams = lin.params(hq, THETA)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    keep_k = {b: [] for b in sample}
    keep_v = {b: [] for b in sample}
    chunk = 4096
    for c0 in range(0, lmax - 1, chunk):  # positions [0, lmax - 1); the query's own row next
        T = min(chunk, lmax - 1 - c0)
        k = synth.normal_bf16((Bn, T, hkv, D), 5000 + c0, dev)
        v = synth.normal_bf16((Bn, T, hkv, D), 9000 + c0, dev)
        B.ps_kv_append_rope(aparams, lin.struct, k, v, None,
                            torch.full((Bn,), c0, dtype=torch.int64, device=dev), T, st)
        for b in sample:
            keep_k[b].append(k[b].cpu())
            keep_v[b].append(v[b].cpu())
    for b, p in enumerate(P):  # nothing past each sequence's own history
        lin.k[b, :, p:].fill_(float("nan"))
        lin.v[b, :, p:].fill_(float("nan"))
    k_new = synth.normal_bf16((Bn, 1, hkv, D), 77, dev)
    v_new = synth.normal_bf16((Bn, 1, hkv, D), 78, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), 79, dev)
    q = q_raw.clone()
    B.ps_kv_append_rope(aparams, lin.struct, k_new, v_new, q.view(Bn, 1, hq, D), pos, 1, st)
    params = B.make_params(hq, hkv, D, 0, 1, THETA)
    out = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_full_attn_workspace_bytes(params, Bn, lmax)), dtype=torch.uint8,
                     device=dev)
    B.ps_full_attn_ref(params, lin.k, lin.v, lmax, q, pos, Bn, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.isfinite(out.float()).all()
    got, gl = f64(out), f64(lse)
    qr, kn, vn = f64(q_raw), f64(k_new), f64(v_new)
    scale = 1 / math.sqrt(D)
    for b in sample:
        p = P[b]
        kr = np.concatenate([torch.cat(keep_k[b])[:p].double().numpy(), kn[b]], axis=0)
        vr = np.concatenate([torch.cat(keep_v[b])[:p].double().numpy(), vn[b]], axis=0)
        k_rot = O.rope_rotate(kr, np.arange(p + 1)[:, None], THETA)
        o, l = O.full_attention_decode(O.rope_rotate(qr[b], p, THETA), k_rot, vr, p, scale)
        assert_close(got[b], o, f"full b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2


@pytest.mark.parametrize("hq,hkv,lp,w,S,rows", [
    (16, 2, 100, 512, 1500, [0, 50, 99, 100, 300, 611, 612, 613, 1000, 1499]),
    (28, 4, 256, 2048, 4096, [255, 1000, 2303, 2304, 2305, 3000, 4095]),
])
def test_decode_equals_prefill_row(cuda_device, hq, hkv, lp, w, S, rows):
    """Decode at position p (ps_decode_step over the prefix + ring store) equals row p of the
    masked prefill over the same sequence, for p in the prefix, in warm-up, at the cap
    (n = L_prefix + W), at the first slide and past it.  The prefill reads Q and K rotated by
    the same append kernel (a linear cache holds every rotated key)."""
    dev = cuda_device
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    k_raw = synth.normal_bf16((1, S, hkv, D), 91, dev)
    v_raw = synth.normal_bf16((1, S, hkv, D), 92, dev)
    q_raw = synth.normal_bf16((1, S, hq, D), 93, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    # prefill: every key rotated at its index (linear cache), every query too
    lin = LinearCache(1, hkv, S, D, dev)
    q_rot = q_raw.clone()
    B.ps_kv_append_rope(lin.params(hq, THETA), lin.struct, k_raw, v_raw, q_rot,
                        torch.zeros(1, dtype=torch.int64, device=dev), S, st)
    k_rot = lin.k.permute(0, 2, 1, 3).contiguous()
    v_lin = lin.v.permute(0, 2, 1, 3).contiguous()
    assert torch.equal(v_lin, v_raw)
    out_p = torch.empty_like(q_raw)
    ws_p = torch.empty(B.ps_prefill_workspace_bytes(params, 1, S), dtype=torch.uint8, device=dev)
    B.ps_masked_prefill_attn(params, q_rot, k_rot, v_lin, 1, S, out_p, None, None, ws_p, st)
    # decode: one sequence per probed row, history [0, p) appended, then one decode step at p
    Bn = len(rows)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    for b, p in enumerate(rows):
        if p:
            B.ps_kv_append_rope(params, _view(cache, b, b + 1), k_raw[:, :p].contiguous(),
                                v_raw[:, :p].contiguous(), None,
                                torch.zeros(1, dtype=torch.int64, device=dev), p, st)
    idx = torch.tensor(rows, device=dev)
    pos = idx.to(torch.int64)
    q = q_raw[0, idx].contiguous()
    out_d = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    B.ps_decode_step(params, cache.struct, k_raw[0, idx].contiguous(), v_raw[0, idx].contiguous(),
                     q, pos, out_d, None, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(q, q_rot[0, idx])  # the same rotation on both paths
    for b, p in enumerate(rows):
        assert_close(f64(out_d[b]), f64(out_p[0, p]), f"decode vs prefill row {p}")
