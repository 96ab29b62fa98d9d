"""GPU parity of the paged store (block pool + per-sequence block tables) against the
float64 oracle, through the C ABI.

Sequences' blocks are scattered over the pool in a seeded random order; a group of
sequences shares one set of prefix blocks (one prompt, pinned once).  Decode must match the
oracle (max_abs <= 2e-2, rel_rms <= 5e-3, lse within 2e-2) and agree with the contiguous
store's decode on the same keys.  Pools start NaN-filled, so a read of a row that was never
written shows up as a non-finite output.
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
from tests.test_gpu_decode import THETA, _oracle_decode_from_history

pytestmark = pytest.mark.gpu

D = 128


def _paged_case(dev, lp, w, positions, share, seed, hq=16, hkv=2):
    """positions[b]: decoded position of sequence b; sequences [0, share) share their prefix
    blocks (and prompt)."""
    Bn = len(positions)
    pre_blocks = -(-lp // 64)
    per_seq = pre_blocks + w // 64
    stride = per_seq + 3  # a little slack: the stride need not be tight
    n_blocks = Bn * per_seq + 5
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_blocks)
    table = np.full((Bn, stride), -1, np.int32)
    for b in range(Bn):
        table[b, :per_seq] = perm[b * per_seq:(b + 1) * per_seq]
    table[1:share, :pre_blocks] = table[0, :pre_blocks]  # one prompt, one set of blocks
    table_d = torch.from_numpy(table).to(dev)
    nan = float("nan")
    k_pool = torch.full((n_blocks, hkv, 64, D), nan, dtype=torch.bfloat16, device=dev)
    v_pool = torch.full_like(k_pool, nan)
    Smax = max(max(positions) + 1, lp)
    k_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed + 1, dev)
    v_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed + 2, dev)
    k_raw[1:share, :lp] = k_raw[0, :lp]
    v_raw[1:share, :lp] = v_raw[0, :lp]
    q_raw = synth.normal_bf16((Bn, hq, D), seed + 3, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    contig = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=nan)
    zero = torch.zeros(1, dtype=torch.int64, device=dev)
    # the shared prompt is written once, through sequence 0's table
    B.ps_kv_append_rope_paged(params, k_pool, v_pool, table_d[:1], 1,
                              k_raw[:1, :lp].contiguous(), v_raw[:1, :lp].contiguous(), None,
                              zero, lp, st)
    for b, p in enumerate(positions):
        first = lp if b < share else 0  # sharing sequences add only their own tokens
        if p >= first:
            B.ps_kv_append_rope_paged(params, k_pool, v_pool, table_d[b:b + 1], 1,
                                      k_raw[b:b + 1, first:p + 1].contiguous(),
                                      v_raw[b:b + 1, first:p + 1].contiguous(), None,
                                      zero + first, p - first + 1, st)
        view = B.make_cache(contig.k_prefix[b:b + 1], contig.v_prefix[b:b + 1],
                            contig.k_ring[b:b + 1], contig.v_ring[b:b + 1], 1)
        B.ps_kv_append_rope(params, view, k_raw[b:b + 1, :p + 1].contiguous(),
                            v_raw[b:b + 1, :p + 1].contiguous(), None, zero, p + 1, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, k_raw[:, :1].contiguous(),
                        v_raw[:, :1].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    out = torch.full((Bn, hq, D), nan, dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), nan, dtype=torch.float32, device=dev)
    B.ps_decode_attn_paged(params, k_pool, v_pool, table_d, Bn, q, pos, out, lse, ws, st)
    out_c = torch.empty_like(out)
    B.ps_decode_attn(params, contig.struct, q, pos, out_c, None, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    qr, kr, vr = f64(q_raw), f64(k_raw), f64(v_raw)
    got, gl = f64(out), f64(lse)
    for b, p in enumerate(positions):
        o, l = _oracle_decode_from_history(B_rope(qr[b], p), kr[b, :p + 1], vr[b, :p + 1], p,
                                           lp, w, 1 / math.sqrt(D))
        assert_close(got[b], o, f"paged b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, (b, p)
    assert np.abs(got - f64(out_c)).max() < 1e-2
    return params, k_pool, v_pool, table_d, pos, q, st


def B_rope(q_b, p):
    import oracle as O
    return O.rope_rotate(q_b, p, THETA)


def test_paged_split_k_schedule_with_shared_prompt_blocks(cuda_device):
    """12 sequences (24 units: stream-K), the first 4 sharing one prompt's blocks;
    L_prefix 100 (a partly filled last prefix block), W 256; in-prompt, warm-up, exact cap
    and wrapped positions."""
    positions = [99, 100, 355, 356, 50, 101, 700, 1000, 2047, 357, 612, 3333]
    _paged_case(cuda_device, 100, 256, positions, share=4, seed=801)


def test_paged_per_unit_schedule(cuda_device):
    """160 sequences (one CTA per unit), prefix of exactly two blocks, W 128."""
    rng = np.random.default_rng(9)
    positions = rng.integers(0, 1500, size=160).tolist()
    _paged_case(cuda_device, 128, 128, positions, share=8, seed=811)


def test_paged_bad_table_entry_is_flagged(cuda_device):
    """An entry outside [0, n_blocks) sets PS_DEV_POS_RANGE in the append (nothing written)
    and in the decode (zeros read)."""
    dev = cuda_device
    params, k_pool, v_pool, table, pos, q, st = _paged_case(dev, 64, 128, [300, 400], share=1,
                                                            seed=821)
    bad = table.clone()
    bad[0, 1] = k_pool.shape[0] + 7  # a ring block of sequence 0
    before = k_pool.clone()
    st.zero_()
    k1 = synth.normal_bf16((1, 1, 2, D), 5, dev)
    p = torch.tensor([64 + 10], dtype=torch.int64, device=dev)  # ring slot 10: entry 1
    B.ps_kv_append_rope_paged(params, k_pool, v_pool, bad[:1], 1, k1, k1, None, p, 1, st)
    torch.cuda.synchronize()
    assert st.item() == B.PS_DEV_POS_RANGE
    assert torch.equal(k_pool.isnan(), before.isnan())
    st.zero_()
    out = torch.empty((2, 16, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, 2)), dtype=torch.uint8, device=dev)
    B.ps_decode_attn_paged(params, k_pool, v_pool, bad, 2, q, pos, out, None, ws, st)
    torch.cuda.synchronize()
    assert st.item() == B.PS_DEV_POS_RANGE


def test_paged_pure_window_step_flow(cuda_device):
    """L_prefix = 0 (no prefix blocks), W = 64 (one ring block): each sequence appends its
    history, then its newest token together with q (rotated in place, bit-identical to the
    contiguous append's rotation), then decodes; held to the oracle."""
    dev = cuda_device
    lp, w, hq, hkv = 0, 64, 16, 2
    positions = [0, 1, 63, 64, 65, 200, 1000]
    Bn = len(positions)
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    n_blocks = Bn + 2
    table = torch.tensor(np.random.default_rng(3).permutation(n_blocks)[:Bn].reshape(Bn, 1),
                         dtype=torch.int32, device=dev)
    nan = float("nan")
    k_pool = torch.full((n_blocks, hkv, 64, D), nan, dtype=torch.bfloat16, device=dev)
    v_pool = torch.full_like(k_pool, nan)
    Smax = max(positions) + 1
    k_raw = synth.normal_bf16((Bn, Smax, hkv, D), 831, dev)
    v_raw = synth.normal_bf16((Bn, Smax, hkv, D), 832, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), 833, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int64, device=dev)
    for b, p in enumerate(positions):
        if p > 0:
            B.ps_kv_append_rope_paged(params, k_pool, v_pool, table[b:b + 1], 1,
                                      k_raw[b:b + 1, :p].contiguous(),
                                      v_raw[b:b + 1, :p].contiguous(), None, zero, p, st)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    k_last = torch.stack([k_raw[b, p] for b, p in enumerate(positions)]).view(Bn, 1, hkv, D)
    v_last = torch.stack([v_raw[b, p] for b, p in enumerate(positions)]).view(Bn, 1, hkv, D)
    q = q_raw.clone()
    B.ps_kv_append_rope_paged(params, k_pool, v_pool, table, Bn, k_last.contiguous(),
                              v_last.contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    q_ref = q_raw.clone()
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    B.ps_kv_append_rope(params, scratch.struct, k_last.contiguous(), v_last.contiguous(),
                        q_ref.view(Bn, 1, hq, D), pos, 1, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    assert torch.equal(q, q_ref)
    out = torch.full((Bn, hq, D), nan, dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), nan, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    B.ps_decode_attn_paged(params, k_pool, v_pool, table, Bn, q, pos, out, lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    qr, kr, vr = f64(q_raw), f64(k_raw), f64(v_raw)
    got, gl = f64(out), f64(lse)
    for b, p in enumerate(positions):
        o, l = _oracle_decode_from_history(B_rope(qr[b], p), kr[b, :p + 1], vr[b, :p + 1], p,
                                           lp, w, 1 / math.sqrt(D))
        assert_close(got[b], o, f"paged lp=0 b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, (b, p)


def test_paged_full_size_b64_w4096(cuda_device):
    """The bench's paged leg at full size: batch 64, 16/2/128, L_prefix 100, W 4096,
    positions drawn in [8192, 131072]; the contiguous store's rows copied into 66 scattered
    blocks per sequence.  Sampled sequences against the oracle, every sequence against the
    contiguous decode."""
    dev = cuda_device
    wl = synth.WORKLOADS["decode_b64_w4096"]
    hq, hkv, lp, w, Bn = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window, wl.batch
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, synth.seed_for(2, 10), dev)
    k_pre = synth.normal_bf16((Bn, lp, hkv, D), synth.seed_for(2, 11), dev)
    v_pre = synth.normal_bf16((Bn, lp, hkv, D), synth.seed_for(2, 12), dev)
    k_win = synth.normal_bf16((Bn, w, hkv, D), synth.seed_for(2, 13), dev)
    v_win = synth.normal_bf16((Bn, w, hkv, D), synth.seed_for(2, 14), dev)
    q_raw = synth.normal_bf16((Bn, hq, D), synth.seed_for(2, 15), dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    B.ps_kv_append_rope(params, cache.struct, k_pre, v_pre, None,
                        torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
    q = q_raw.clone()
    # window positions p - W + 1 .. p; q rotated with the newest token
    B.ps_kv_append_rope(params, cache.struct, k_win[:, :w - 1].contiguous(),
                        v_win[:, :w - 1].contiguous(), None, pos - (w - 1), w - 1, st)
    B.ps_kv_append_rope(params, cache.struct, k_win[:, w - 1:].contiguous(),
                        v_win[:, w - 1:].contiguous(), q.view(Bn, 1, hq, D), pos, 1, st)
    pre_blocks, ring_blocks = -(-lp // 64), w // 64
    per_seq = pre_blocks + ring_blocks
    n_blocks = Bn * per_seq
    perm = torch.from_numpy(np.random.default_rng(21).permutation(n_blocks)).to(dev)
    table = perm.view(Bn, per_seq).to(torch.int32)
    nan = float("nan")
    k_pool = torch.full((n_blocks, hkv, 64, D), nan, dtype=torch.bfloat16, device=dev)
    v_pool = torch.full_like(k_pool, nan)
    for src_pre, src_ring, pool in ((cache.k_prefix, cache.k_ring, k_pool),
                                    (cache.v_prefix, cache.v_ring, v_pool)):
        pre = torch.full((Bn, hkv, pre_blocks * 64, D), nan, dtype=torch.bfloat16, device=dev)
        pre[:, :, :lp] = src_pre
        blocks = torch.cat([pre.view(Bn, hkv, pre_blocks, 64, D),
                            src_ring.view(Bn, hkv, ring_blocks, 64, D)], dim=2)
        pool[table.long().view(-1)] = blocks.permute(0, 2, 1, 3, 4).reshape(n_blocks, hkv, 64, D)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    out = torch.full((Bn, hq, D), nan, dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), nan, dtype=torch.float32, device=dev)
    B.ps_decode_attn_paged(params, k_pool, v_pool, table, Bn, q, pos, out, lse, ws, st)
    out_c = torch.empty_like(out)
    B.ps_decode_attn(params, cache.struct, q, pos, out_c, None, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    assert torch.isfinite(out.float()).all()
    assert (out.float() - out_c.float()).abs().max().item() < 1e-2
    P = pos.cpu().numpy()
    kp, vp, kw, vw, qr = f64(k_pre), f64(v_pre), f64(k_win), f64(v_win), f64(q_raw)
    got, gl = f64(out), f64(lse)
    for b in (0, 21, 42, 63):
        p = int(P[b])
        vis = O.visible_positions(p, lp, w)
        base = p - (w - 1)
        kr = np.stack([kp[b, x] if x < lp else kw[b, x - base] for x in vis])
        vr = np.stack([vp[b, x] if x < lp else vw[b, x - base] for x in vis])
        o, l = O.attend_gqa(O.rope_rotate(qr[b], p, THETA), O.rope_rotate(kr, vis[:, None], THETA),
                            vr, 1 / math.sqrt(D))
        assert_close(got[b], o, f"paged full size b={b}")
        assert np.abs(gl[b] - l).max() < 2e-2
