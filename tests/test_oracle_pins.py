"""Pins for the float64 oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers the pages
print (tests/golden/pages_numbers.json), closed forms, an independent library routine
(torch scaled_dot_product_attention / logsumexp in float64), a complex-number form of
RoPE, or brute force on tiny inputs.  A plausible slip in the oracle (an off-by-one
window, a wrong RoPE sign, a swapped GQA map, a dropped max term) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, causal=False):
    """torch SDPA in float64 with its own GQA mapping.  q [Sq,Hq,D], k/v [Sk,Hkv,D]."""
    tq = torch.from_numpy(np.ascontiguousarray(q)).permute(1, 0, 2)[None]
    tk = torch.from_numpy(np.ascontiguousarray(k)).permute(1, 0, 2)[None]
    tv = torch.from_numpy(np.ascontiguousarray(v)).permute(1, 0, 2)[None]
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=True)
    return out[0].permute(1, 0, 2).numpy()


# ------------------------------------------------------------ pages' numbers
def test_memory_cap_printed_value():
    """eq. L_total: prefix 100 + window 4096 -> at most 4196 visible keys, for any n."""
    for case in _golden()["memory_cap"]:
        lp, w, cap = case["l_prefix"], case["window"], case["l_total"]
        for p in (lp + w - 1, lp + w, 10_000, 131_071):
            assert len(O.visible_positions(p, lp, w)) == cap


def test_kv_bytes_formula_printed_values():
    for case in _golden()["kv_bytes_per_token"]:
        b = O.kv_bytes_per_token(case["n_layers"], case["n_kv_heads"], case["head_dim"],
                                 case["bytes_per_elem"])
        assert round(b / 1024) == case["approx_kib"] or math.floor(b / 1000) == case["approx_kib"]
        if "tokens_1m_approx_gb" in case:
            assert math.floor(b * 1_000_000 / 1e9) == case["tokens_1m_approx_gb"]
        if "tokens_100k_approx_gb" in case:
            assert math.floor(b * 100_000 / 1e8) / 10 == case["tokens_100k_approx_gb"]


def test_truncated_context_printed_split():
    c = _golden()["truncated_backprop"]
    first_sent, first_loss, sent, loss = O.truncated_context(c["rollout_tokens"], c["window"])
    assert sent == c["sent"] and loss == c["loss"]
    assert first_loss - first_sent == c["context"]
    assert c["rollout_tokens"] - first_sent == c["sent"]


# ------------------------------------------------------------- visibility
@settings(max_examples=300, deadline=None)
@given(lp=st.integers(0, 40), w=st.integers(1, 40), p=st.integers(0, 200))
def test_visible_count_closed_form(lp, w, p):
    """|V(p)| = min(n, L_prefix + W) with n = p + 1 (eq. L_total and the warm-up note)."""
    vis = O.visible_positions(p, lp, w)
    assert len(vis) == min(p + 1, lp + w)
    assert len(set(vis.tolist())) == len(vis)  # no key counted twice
    assert vis.max() == p  # every query sees itself
    # the prefix is pinned: every k < min(L_prefix, n) is visible
    assert set(range(min(lp, p + 1))) <= set(vis.tolist())
    # the most recent min(W, n) positions are visible
    assert set(range(max(0, p - w + 1), p + 1)) <= set(vis.tolist())


def test_visible_positions_tiny_by_hand():
    # L_prefix=2, W=3, query p=7: prefix {0,1}, window {5,6,7}
    assert O.visible_positions(7, 2, 3).tolist() == [0, 1, 5, 6, 7]
    # warm-up: p=4 -> n=5 = L_prefix+W -> everything
    assert O.visible_positions(4, 2, 3).tolist() == [0, 1, 2, 3, 4]
    # pure sliding window
    assert O.visible_positions(7, 0, 3).tolist() == [5, 6, 7]


# ------------------------------------------------------------------ RoPE
def test_rope_matches_complex_rotation():
    """Rotate-half RoPE equals multiplying z = x1 + i*x2 by exp(i * p * inv_f)."""
    d, theta = 128, 1.0e6
    x = _rand((5, 3, d), 1)
    pos = np.array([0, 1, 611, 131071, 262143], dtype=np.int64)[:, None] * np.ones((1, 3), np.int64)
    got = O.rope_rotate(x, pos, theta)
    i = np.arange(d // 2)
    inv = theta ** (-(2.0 * i) / d)
    z = (x[..., : d // 2] + 1j * x[..., d // 2:]) * np.exp(1j * pos[..., None] * inv)
    want = np.concatenate([z.real, z.imag], axis=-1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def test_rope_inv_freq_closed_form():
    d, theta = 128, 1.0e6
    f = O.rope_inv_freq(d, theta)
    assert f.shape == (64,)
    assert f[0] == 1.0
    np.testing.assert_allclose(f[1:] / f[:-1], theta ** (-2.0 / d), rtol=1e-13)
    np.testing.assert_allclose(f[-1], theta ** (-(d - 2) / d), rtol=1e-13)


def test_rope_relative_position_identity():
    """<R_a q, R_b k> = <q, R_{b-a} k>: scores depend only on the position gap."""
    d, theta = 128, 1.0e6
    q, k = _rand((d,), 2), _rand((d,), 3)
    for a, b in [(0, 5), (100, 4196), (8192, 131071), (250000, 262143)]:
        lhs = O.rope_rotate(q, a, theta) @ O.rope_rotate(k, b, theta)
        rhs = q @ O.rope_rotate(k, b - a, theta)
        assert abs(lhs - rhs) < 1e-8 * (1 + abs(rhs))


def test_rope_identity_at_zero_and_norm():
    x = _rand((4, 128), 4)
    np.testing.assert_array_equal(O.rope_rotate(x, 0, 1e6), x)
    y = O.rope_rotate(x, 123457, 1e6)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


# ------------------------------------------------------------- attention
def test_attend_tiny_bruteforce_loops():
    """Pure-Python nested-loop softmax on a tiny GQA shape."""
    hq, hkv, d, n = 4, 2, 3, 5
    q, k, v = _rand((hq, d), 5), _rand((n, hkv, d), 6), _rand((n, hkv, d), 7)
    scale = 0.7
    out, lse = O.attend_gqa(q, k, v, scale)
    for h in range(hq):
        kv = h // (hq // hkv)
        s = [sum(q[h][c] * k[j][kv][c] for c in range(d)) * scale for j in range(n)]
        z = sum(math.exp(x) for x in s)
        for c in range(d):
            o = sum(math.exp(s[j]) / z * v[j][kv][c] for j in range(n))
            assert abs(o - out[h][c]) < 1e-12
        assert abs(math.log(z) - lse[h]) < 1e-12


def test_lse_matches_torch_logsumexp():
    hq, hkv, d, n = 8, 2, 16, 40
    q, k, v = _rand((hq, d), 8) * 4, _rand((n, hkv, d), 9) * 4, _rand((n, hkv, d), 10)
    scale = 0.25
    _, lse = O.attend_gqa(q, k, v, scale)
    kk = torch.from_numpy(k).repeat_interleave(hq // hkv, dim=1)  # [n, hq, d]
    s = torch.einsum("hd,nhd->hn", torch.from_numpy(q), kk) * scale
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("lp,w,S", [(3, 5, 8), (0, 20, 20), (7, 30, 25), (16, 16, 32)])
def test_warmup_equals_full_causal(lp, w, S):
    """n <= L_prefix + W (or W >= n): the mask is plain causal attention (warm-up note)."""
    assert S <= lp + w
    hq, hkv, d = 8, 2, 16
    Q, K, V = _rand((S, hq, d), 11), _rand((S, hkv, d), 12), _rand((S, hkv, d), 13)
    scale = 1 / math.sqrt(d)
    got, _ = O.prefill_reference(Q, K, V, lp, w, scale)
    want = _sdpa(Q, K, V, scale, causal=True)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_pure_sliding_window_is_prefixless_case():
    """L_prefix = 0 recovers the textbook sliding window over the last W keys."""
    S, w, hq, hkv, d = 40, 7, 4, 1, 8
    Q, K, V = _rand((S, hq, d), 14), _rand((S, hkv, d), 15), _rand((S, hkv, d), 16)
    scale = 0.3
    got, _ = O.prefill_reference(Q, K, V, 0, w, scale)
    for i in range(S):
        lo = max(0, i - w + 1)
        want = _sdpa(Q[i:i + 1], K[lo:i + 1], V[lo:i + 1], scale)[0]
        np.testing.assert_allclose(got[i], want, rtol=0, atol=1e-12)


def test_prefix_sliding_equals_sdpa_over_two_slices():
    """Beyond warm-up each row equals attention over K[:L_prefix] ++ K[i-W+1 : i+1]."""
    S, lp, w, hq, hkv, d = 64, 5, 9, 8, 2, 16
    Q, K, V = _rand((S, hq, d), 17), _rand((S, hkv, d), 18), _rand((S, hkv, d), 19)
    scale = 1 / 4
    rows = list(range(lp + w, S))
    got, _ = O.prefill_reference(Q, K, V, lp, w, scale, rows=rows)
    for r, i in enumerate(rows):
        kk = np.concatenate([K[:lp], K[i - w + 1:i + 1]])
        vv = np.concatenate([V[:lp], V[i - w + 1:i + 1]])
        want = _sdpa(Q[i:i + 1], kk, vv, scale)[0]
        np.testing.assert_allclose(got[r], want, rtol=0, atol=1e-12)


def test_full_attention_decode_equals_causal_last_row():
    S, hq, hkv, d = 30, 4, 2, 8
    Q, K, V = _rand((S, hq, d), 20), _rand((S, hkv, d), 21), _rand((S, hkv, d), 22)
    got, _ = O.full_attention_decode(Q[S - 1], K, V, S - 1, 0.5)
    want = _sdpa(Q, K, V, 0.5, causal=True)[S - 1]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ------------------------------------------------------- ring simulator
@pytest.mark.parametrize("lp,w,steps", [(4, 6, 40), (0, 5, 23), (10, 1, 30), (3, 17, 19)])
def test_ring_keeps_exactly_the_visible_set(lp, w, steps):
    """Hard eviction never drops a visible key, and storage is capped at L_prefix + W."""
    hkv, d = 2, 4
    ring = O.RingKVCache(lp, w, hkv, d, 1e6)
    for p in range(steps):
        ring.append(p, _rand((hkv, d), 100 + p), _rand((hkv, d), 200 + p))
        vis = O.visible_positions(p, lp, w).tolist()
        assert [e[2] for e in ring.visible_entries(p)] == vis
        held = ring.held_positions()
        assert len(held) <= lp + w
        assert held == vis  # everything still stored is visible (nothing stale kept)


@settings(max_examples=200, deadline=None)
@given(lp=st.integers(0, 12), w=st.integers(1, 12), p=st.integers(0, 60))
def test_ring_descriptor_closed_form(lp, w, p):
    """Descriptor read off the slots equals the closed form of the visible ranges."""
    ring = O.RingKVCache(lp, w, 1, 2, 1e6)
    z = np.zeros((1, 2))
    for t in range(p + 1):
        ring.append(t, z, z)
    pre_len, s0, l0, l1 = ring.descriptor(p)
    n = p + 1
    wstart = max(lp, n - w)
    win = n - wstart
    assert pre_len == min(n, lp)
    assert pre_len + l0 + l1 == min(n, lp + w)
    if win > 0:
        assert s0 == (wstart - lp) % w
        assert l0 == min(win, w - s0)
        assert l1 == win - l0
    else:
        assert (s0, l0, l1) == (0, 0, 0)


def test_continue_pe_ring_decode_equals_recomputed_rope():
    """Keys rotated once at append (Continue PE) give the same output as rotating every
    cached raw key again at its original absolute position at each step."""
    lp, w, hq, hkv, d, theta = 3, 5, 4, 2, 8, 1e6
    steps = 20
    raw_k = _rand((steps, hkv, d), 30)
    vals = _rand((steps, hkv, d), 31)
    qs = _rand((steps, hq, d), 32)
    ring = O.RingKVCache(lp, w, hkv, d, theta)
    for p in range(steps):
        ring.append(p, raw_k[p], vals[p])
        ents = ring.visible_entries(p)
        k_once = np.stack([e[3] for e in ents])
        v_once = np.stack([e[4] for e in ents])
        q = O.rope_rotate(qs[p], p, theta)
        out_ring, _ = O.attend_gqa(q, k_once, v_once, 0.35)
        k_re = O.rope_rotate(raw_k[: p + 1], np.arange(p + 1)[:, None], theta)
        out_def, _ = O.decode_reference(q, k_re, vals, p, lp, w, 0.35)
        np.testing.assert_allclose(out_ring, out_def, rtol=0, atol=1e-12)


# -------------------------------------------------------------- tile plan
def _interval_counts(seq, lp, w, bq, bk):
    """Independent count: per row, visible columns are two intervals
    [0, min(lp, i+1)) and [max(lp, i-w+1), i+1); intersect them with each k tile."""
    nq, nk = -(-seq // bq), -(-seq // bk)
    out = np.zeros((nq, nk), np.int64)
    for i in range(seq):
        ivs = [(0, min(lp, i + 1)), (max(lp, i - w + 1), i + 1)]
        for kt in range(nk):
            a, b = kt * bk, min(seq, (kt + 1) * bk)
            out[i // bq, kt] += sum(max(0, min(b, hi) - max(a, lo)) for lo, hi in ivs)
    return out


@pytest.mark.parametrize("seq,lp,w,bq,bk", [(300, 20, 50, 32, 32), (257, 0, 64, 64, 32),
                                           (512, 128, 128, 128, 128), (200, 7, 500, 16, 64)])
def test_tile_counts_match_interval_arithmetic(seq, lp, w, bq, bk):
    np.testing.assert_array_equal(O.tile_counts(seq, lp, w, bq, bk),
                                  _interval_counts(seq, lp, w, bq, bk))


def test_tile_counts_total_is_sum_of_visible_counts():
    seq, lp, w = 1000, 33, 100
    total = O.tile_counts(seq, lp, w, 64, 64).sum()
    assert total == sum(min(i + 1, lp + w) for i in range(seq))


def test_tile_plan_window_covering_sequence_is_causal_triangle():
    """W >= seq: plan = lower triangle, diagonal tiles PARTIAL, the rest FULL."""
    seq, b = 512, 64
    plan = O.tile_plan(seq, 0, seq, b, b)
    nt = seq // b
    want = [(qt, kt, O.TILE_PARTIAL if kt == qt else O.TILE_FULL)
            for qt in range(nt) for kt in range(qt + 1)]
    assert [tuple(r) for r in plan.tolist()] == want


def test_tile_plan_ragged_tail_is_partial():
    plan = O.tile_plan(300, 0, 300, 128, 128)
    flags = {(q, k): f for q, k, f in plan.tolist()}
    assert flags[(2, 0)] == O.TILE_PARTIAL  # rows 256..299 only: not a full 128-row tile
    assert flags[(1, 0)] == O.TILE_FULL


def test_tile_plan_truncated_backprop_context_skips():
    """The 4W training context of the §截断回传 example shape (S=8192, W=2048) with a
    256-token prefix: skip/partial/full split from the independent interval count."""
    seq, lp, w, b = 8192, 256, 2048, 128
    plan = O.tile_plan(seq, lp, w, b, b)
    cnt = _interval_counts(seq, lp, w, b, b)
    n_full = int((cnt == b * b).sum())
    n_part = int(((cnt > 0) & (cnt < b * b)).sum())
    assert (plan[:, 2] == O.TILE_FULL).sum() == n_full
    assert (plan[:, 2] == O.TILE_PARTIAL).sum() == n_part
    assert (n_full, n_part, 64 * 64 - n_full - n_part) == (935, 110, 3051)


def test_tile_plan_one_hidden_pair_is_partial():
    """Rows {2,3} x cols {0,1}, W=3: only (3, 0) is hidden -> PARTIAL, not FULL."""
    plan = O.tile_plan(4, 0, 3, 2, 2)
    assert [tuple(r) for r in plan.tolist()] == [(0, 0, O.TILE_PARTIAL), (1, 0, O.TILE_PARTIAL),
                                                 (1, 1, O.TILE_PARTIAL)]


@pytest.mark.parametrize("seq,lp,w,bq,bk", [(300, 20, 50, 32, 32), (257, 0, 64, 64, 32),
                                           (640, 100, 130, 64, 64)])
def test_tile_plan_flags_from_interval_counts(seq, lp, w, bq, bk):
    cnt = _interval_counts(seq, lp, w, bq, bk)
    want = [(q, k, O.TILE_FULL if c == bq * bk else O.TILE_PARTIAL)
            for q in range(cnt.shape[0]) for k in range(cnt.shape[1]) for c in [cnt[q, k]] if c > 0]
    assert [tuple(r) for r in O.tile_plan(seq, lp, w, bq, bk).tolist()] == want


# ------------------------------------------------------- masked prefill backward
def _autograd_grads(Q, K, V, dO, lp, w, scale):
    """Gradients from torch autograd through SDPA in float64 with an explicit boolean
    mask built from the 0-indexed eq. A(i) and torch's own GQA expansion."""
    S = Q.shape[0]
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    mask = (j <= i) & ((j < lp) | (j > i - w))
    tq = torch.from_numpy(Q).permute(1, 0, 2)[None].requires_grad_(True)
    tk = torch.from_numpy(K).permute(1, 0, 2)[None].requires_grad_(True)
    tv = torch.from_numpy(V).permute(1, 0, 2)[None].requires_grad_(True)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, scale=scale, enable_gqa=True)
    out.backward(torch.from_numpy(dO).permute(1, 0, 2)[None])
    return [t.grad[0].permute(1, 0, 2).numpy() for t in (tq, tk, tv)]


@pytest.mark.parametrize("S,lp,w,hq,hkv", [(24, 3, 5, 4, 2), (30, 0, 7, 6, 2), (17, 17, 1, 2, 1),
                                          (20, 4, 40, 8, 1), (33, 2, 1, 3, 3)])
def test_prefill_backward_matches_autograd(S, lp, w, hq, hkv):
    d, scale = 8, 0.37
    Q, K, V = _rand((S, hq, d), 40), _rand((S, hkv, d), 41), _rand((S, hkv, d), 42)
    dO = _rand((S, hq, d), 43)
    dq, dk, dv = O.prefill_backward_reference(Q, K, V, dO, lp, w, scale)
    wq, wk, wv = _autograd_grads(Q, K, V, dO, lp, w, scale)
    for got, want in ((dq, wq), (dk, wk), (dv, wv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_prefill_backward_central_differences_of_forward():
    """Brute force: d/dx of L = sum(dO * O) by central differences of the forward oracle,
    for every element of a tiny Q, K and V."""
    S, lp, w, hq, hkv, d, scale = 7, 2, 3, 2, 1, 3, 0.8
    Q, K, V = _rand((S, hq, d), 44), _rand((S, hkv, d), 45), _rand((S, hkv, d), 46)
    dO = _rand((S, hq, d), 47)
    dq, dk, dv = O.prefill_backward_reference(Q, K, V, dO, lp, w, scale)

    def loss(q, k, v):
        return float((O.prefill_reference(q, k, v, lp, w, scale)[0] * dO).sum())

    eps = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        args = [Q, K, V]
        num = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            hi = [a.copy() for a in args]
            lo = [a.copy() for a in args]
            hi[which][idx] += eps
            lo[which][idx] -= eps
            num[idx] = (loss(*hi) - loss(*lo)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=0, atol=1e-7)


def test_prefill_backward_closed_form_sums():
    """Each softmax row sums to one, so sum_j dV_j = sum_i dO_i over a KV head's group,
    and each dS row sums to zero, so sum_j dK_j = 0."""
    S, lp, w, hq, hkv, d = 50, 6, 11, 6, 2, 16
    Q, K, V = _rand((S, hq, d), 48), _rand((S, hkv, d), 49), _rand((S, hkv, d), 50)
    dO = _rand((S, hq, d), 51)
    _, dk, dv = O.prefill_backward_reference(Q, K, V, dO, lp, w, 0.25)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, rtol=0, atol=1e-12)
    want = dO.reshape(S, hkv, hq // hkv, d).sum(axis=(0, 2))
    np.testing.assert_allclose(dv.sum(axis=0), want, rtol=0, atol=1e-12)


def test_prefill_backward_selected_rows_and_keys():
    """Selecting rows/keys returns exactly those rows of the full gradients (prefix keys,
    window keys, the last key; first, middle and last rows)."""
    S, lp, w, hq, hkv, d = 40, 5, 8, 4, 2, 8
    Q, K, V = _rand((S, hq, d), 52), _rand((S, hkv, d), 53), _rand((S, hkv, d), 54)
    dO = _rand((S, hq, d), 55)
    fq, fk, fv = O.prefill_backward_reference(Q, K, V, dO, lp, w, 0.5)
    rows, keys = [0, 17, 39], [0, 4, 5, 20, 39]
    sq, sk, sv = O.prefill_backward_reference(Q, K, V, dO, lp, w, 0.5, rows=rows, keys=keys)
    np.testing.assert_allclose(sq, fq[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(sk, fk[keys], rtol=0, atol=1e-13)
    np.testing.assert_allclose(sv, fv[keys], rtol=0, atol=1e-13)


# ------------------------------------------------------------------- Reset PE
def test_reset_pe_positions_by_hand():
    """L_prefix 3, W 4, query at 10: keys 0,1,2 keep their ids, window 7..10 -> 3..6."""
    vis, ids, q_id = O.reset_pe_positions(10, 3, 4)
    assert vis.tolist() == [0, 1, 2, 7, 8, 9, 10]
    assert ids.tolist() == [0, 1, 2, 3, 4, 5, 6]
    assert q_id == 6


def _continue_pe(q_raw, k_raw, v, p, lp, w, theta, scale):
    vis = O.visible_positions(p, lp, w)
    q = O.rope_rotate(q_raw, p, theta)
    k = O.rope_rotate(k_raw[vis], vis[:, None], theta)
    return O.attend_gqa(q, k, v[vis], scale)


@pytest.mark.parametrize("lp,w,p", [(5, 20, 10), (5, 20, 24), (0, 8, 30), (0, 1, 9)])
def test_reset_pe_equals_continue_pe_without_renumbering_gap(lp, w, p):
    """Warm-up (nothing evicted: ids are the absolute positions) and L_prefix = 0 (only
    relative offsets inside the window matter) give Continue PE exactly."""
    hq, hkv, d = 4, 2, 16
    q, k, v = _rand((hq, d), 60), _rand((p + 1, hkv, d), 61), _rand((p + 1, hkv, d), 62)
    got, gl = O.reset_pe_decode_reference(q, k, v, p, lp, w, 1e4, 0.3)
    want, wl = _continue_pe(q, k, v, p, lp, w, 1e4, 0.3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)
    np.testing.assert_allclose(gl, wl, rtol=0, atol=1e-10)


def test_reset_pe_differs_from_continue_pe_after_eviction():
    """After eviction with a prefix, the prefix-to-query offsets change: results differ."""
    hq, hkv, d, lp, w, p = 4, 2, 16, 4, 6, 40
    q, k, v = _rand((hq, d), 63), _rand((p + 1, hkv, d), 64), _rand((p + 1, hkv, d), 65)
    got, _ = O.reset_pe_decode_reference(q, k, v, p, lp, w, 100.0, 0.5)
    want, _ = _continue_pe(q, k, v, p, lp, w, 100.0, 0.5)
    assert np.abs(got - want).max() > 1e-3


def test_reset_pe_bruteforce_rotation_matrices():
    """Tiny case with explicit 2x2 rotation blocks and a nested-loop softmax."""
    hq, hkv, d, lp, w, p, theta, scale = 2, 1, 4, 2, 3, 9, 50.0, 0.7
    q, k, v = _rand((hq, d), 66), _rand((p + 1, hkv, d), 67), _rand((p + 1, hkv, d), 68)
    keys = [0, 1, 7, 8, 9]                # prefix 0,1; window 7,8,9
    ids = {0: 0, 1: 1, 7: 2, 8: 3, 9: 4}  # window renumbered after the prefix
    qid = 4

    def rot(x, pos):
        y = np.empty(d)
        for i in range(d // 2):
            a = pos * theta ** (-2.0 * i / d)
            c, s_ = math.cos(a), math.sin(a)
            y[i] = x[i] * c - x[i + d // 2] * s_
            y[i + d // 2] = x[i + d // 2] * c + x[i] * s_
        return y

    got, _ = O.reset_pe_decode_reference(q, k, v, p, lp, w, theta, scale)
    for h in range(hq):
        qr = rot(q[h], qid)
        sc = [scale * float(qr @ rot(k[j, 0], ids[j])) for j in keys]
        m = max(sc)
        e = [math.exp(x - m) for x in sc]
        want = sum(ei * v[j, 0] for ei, j in zip(e, keys)) / sum(e)
        np.testing.assert_allclose(got[h], want, rtol=0, atol=1e-12)


def test_reset_pe_equals_shifted_query_for_prefix_keys():
    """Relative form of RoPE: Reset PE scores against window keys equal Continue PE's, and
    against prefix keys equal Continue PE's with the query moved to L_prefix + |win| - 1."""
    hq, hkv, d, lp, w, p, theta = 2, 1, 8, 3, 5, 30, 1e3
    q, k = _rand((hq, d), 69), _rand((p + 1, hkv, d), 70)
    vis, ids, qid = O.reset_pe_positions(p, lp, w)
    kr = O.rope_rotate(k[vis], vis[:, None], theta)[:, 0]   # Continue-PE cached keys
    reset = O.rope_rotate(q, qid, theta) @ O.rope_rotate(k[vis], ids[:, None], theta)[:, 0].T
    cont = O.rope_rotate(q, p, theta) @ kr.T
    moved = O.rope_rotate(q, lp + w - 1, theta) @ kr.T
    pre = vis < lp
    np.testing.assert_allclose(reset[:, ~pre], cont[:, ~pre], rtol=0, atol=1e-10)
    np.testing.assert_allclose(reset[:, pre], moved[:, pre], rtol=0, atol=1e-10)


# ------------------------------------------------------------ appended prefix
def test_pinned_visible_by_hand():
    """L_prefix 2, W 3, promoted {5, 6}: at p = 12 the visible keys are 0, 1, 5, 6, 10..12;
    at p = 7 the promoted tokens are still in the window (no double count)."""
    assert O.pinned_visible_positions(12, 2, 3, [5, 6]).tolist() == [0, 1, 5, 6, 10, 11, 12]
    assert O.pinned_visible_positions(7, 2, 3, [5, 6]).tolist() == [0, 1, 5, 6, 7]
    assert O.pinned_visible_positions(4, 2, 3, [5, 6]).tolist() == [0, 1, 2, 3, 4]


@given(st.integers(0, 20), st.integers(1, 30), st.integers(0, 120),
       st.lists(st.integers(0, 150), max_size=12))
@settings(max_examples=150, deadline=None)
def test_pinned_visible_closed_form(lp, w, p, pinned):
    """Count = |V(p)| + #{promoted t <= p outside V(p)}; no pins = eq. A(i)'s set."""
    got = O.pinned_visible_positions(p, lp, w, pinned)
    base = set(O.visible_positions(p, lp, w).tolist())
    extra = {t for t in pinned if t <= p} - base
    assert len(got) == min(p + 1, lp + w) + len(extra)
    assert O.pinned_visible_positions(p, lp, w, []).tolist() == sorted(base)
    assert np.all(np.diff(got) > 0)


def test_pinned_decode_equals_sdpa_over_the_union():
    hq, hkv, d, lp, w, p = 4, 2, 16, 3, 5, 40
    q, k, v = _rand((hq, d), 71), _rand((p + 1, hkv, d), 72), _rand((p + 1, hkv, d), 73)
    pinned = [10, 11, 12, 30, 38]
    got, _ = O.pinned_decode_reference(q, k, v, p, lp, w, pinned, 0.25)
    keys = sorted(set(range(lp)) | {10, 11, 12, 30} | set(range(p - w + 1, p + 1)))
    want = _sdpa(q[None], k[keys], v[keys], 0.25)[0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
