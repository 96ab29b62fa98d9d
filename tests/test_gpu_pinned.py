"""GPU checks of appending tokens to the pinned prefix at run time (ps_kv_pin) and of the
decode that reads them (ps_decode_attn_pinned), through the C ABI.

Byte work is bit-exact: promoted rows equal the ring rows they were copied from.  Decode is
held to the oracle (pinned_decode_reference: eq. A(i)'s visible set united with the promoted
positions) at max_abs <= 2e-2, rel_rms <= 5e-3, lse within 2e-2.  Stores start NaN-filled.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from tests.gpu_util import assert_close, f64

pytestmark = pytest.mark.gpu

D = 128
THETA = 1.0e6


class _Store:
    """Prefix store with room for promoted tokens, per-sequence rings, pin metadata."""

    def __init__(self, dev, Bn, hkv, lp, w, lcap):
        nan = float("nan")
        self.lp, self.w, self.lcap = lp, w, lcap
        self.k_pre = torch.full((Bn, hkv, lcap, D), nan, dtype=torch.bfloat16, device=dev)
        self.v_pre = torch.full_like(self.k_pre, nan)
        self.k_ring = torch.full((Bn, hkv, w, D), nan, dtype=torch.bfloat16, device=dev)
        self.v_ring = torch.full_like(self.k_ring, nan)
        self.pin_count = torch.zeros(Bn, dtype=torch.int32, device=dev)
        self.pin_pos = torch.full((Bn, lcap - lp), -1, dtype=torch.int64, device=dev)

    def full(self, b0, b1):
        return B.make_cache(self.k_pre[b0:b1], self.v_pre[b0:b1], self.k_ring[b0:b1],
                            self.v_ring[b0:b1], b1 - b0)

    def linear(self, b0, b1):
        return B.make_cache(self.k_pre[b0:b1], self.v_pre[b0:b1], None, None, b1 - b0)

    def ring_only(self, b0, b1):
        return B.make_cache(None, None, self.k_ring[b0:b1], self.v_ring[b0:b1], b1 - b0)


def _run(dev, hq, hkv, lp, w, lcap, plans, seed):
    """plans[b] = (events, p): events are ('upto', a) appends through position a, or
    ('pin', t0, t1) promotions; p is the decoded position.  Returns everything checked."""
    Bn = len(plans)
    Smax = max(p for _, p in plans) + 1
    params = B.make_params(hq, hkv, D, lp, w, THETA)
    lin = B.make_params(hq, hkv, D, lcap, 1, THETA)  # prompt fill of the wider prefix store
    k_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed, dev)
    v_raw = synth.normal_bf16((Bn, Smax, hkv, D), seed + 1, dev)
    q_raw = synth.normal_bf16((Bn, hq, D), seed + 2, dev)
    S = _Store(dev, Bn, hkv, lp, w, lcap)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    one = lambda v: torch.tensor([v], dtype=torch.int64, device=dev)  # noqa: E731
    B.ps_kv_append_rope(lin, S.linear(0, Bn), k_raw[:, :lp].contiguous(),
                        v_raw[:, :lp].contiguous(), None,
                        torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
    copies = []  # (b, row, ring_k_row, ring_v_row) expected after each pin
    pinned = [[] for _ in range(Bn)]
    for b, (events, p) in enumerate(plans):
        cur = lp - 1
        for ev in events + [("upto", p)]:
            if ev[0] == "upto":
                a = ev[1]
                if a > cur:
                    B.ps_kv_append_rope(params, S.ring_only(b, b + 1),
                                        k_raw[b:b + 1, cur + 1:a + 1].contiguous(),
                                        v_raw[b:b + 1, cur + 1:a + 1].contiguous(), None,
                                        one(cur + 1), a - cur, st)
                    cur = a
            else:
                _, t0, t1 = ev
                base = int(S.pin_count[b].item())
                for i, t in enumerate(range(t0, t1)):
                    slot = (t - lp) % w
                    copies.append((b, lp + base + i, S.k_ring[b, :, slot].clone(),
                                   S.v_ring[b, :, slot].clone()))
                B.ps_kv_pin(params, S.full(b, b + 1), lcap, S.pin_count[b:b + 1],
                            S.pin_pos[b:b + 1], one(t0), one(t1), one(cur), st)
                pinned[b].extend(range(t0, t1))
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    for b, row, kr, vr in copies:
        assert torch.equal(S.k_pre[b, :, row], kr) and torch.equal(S.v_pre[b, :, row], vr)
    assert S.pin_count.cpu().tolist() == [len(x) for x in pinned]
    for b in range(Bn):
        assert S.pin_pos[b, :len(pinned[b])].cpu().tolist() == pinned[b]

    pos = torch.tensor([p for _, p in plans], dtype=torch.int64, device=dev)
    q = q_raw.clone()
    scratch_k = torch.zeros((Bn, 1, hkv, D), dtype=torch.bfloat16, device=dev)
    tmp = B.make_cache(None, None, torch.empty_like(S.k_ring), torch.empty_like(S.v_ring), Bn)
    # rotate q at its position (through a throwaway ring)
    B.ps_kv_append_rope(params, tmp, scratch_k, scratch_k, q.view(Bn, 1, hq, D), pos, 1, st)
    out = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, B.ps_decode_pinned_workspace_bytes(params, Bn, lcap)),
                     dtype=torch.uint8, device=dev)
    B.ps_decode_attn_pinned(params, S.full(0, Bn), lcap, S.pin_count, S.pin_pos, q, pos, out,
                            lse, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    qr, kr, vr = f64(q_raw), f64(k_raw), f64(v_raw)
    got, gl = f64(out), f64(lse)
    for b, (_, p) in enumerate(plans):
        vis = O.pinned_visible_positions(p, lp, w, pinned[b])
        k_rot = np.zeros_like(kr[b, :p + 1])
        k_rot[vis] = O.rope_rotate(kr[b, vis], vis[:, None], THETA)
        o, l = O.pinned_decode_reference(O.rope_rotate(qr[b], p, THETA), k_rot, vr[b, :p + 1],
                                         p, lp, w, pinned[b], 1 / math.sqrt(D))
        assert_close(got[b], o, f"pinned b={b} p={p}")
        assert np.abs(gl[b] - l).max() < 2e-2, (b, p)
    return S, st


def test_pinned_tokens_survive_eviction(cuda_device):
    lp, w, lcap = 100, 256, 700
    plans = [
        ([("upto", 400), ("pin", 200, 260), ("upto", 900), ("pin", 700, 705)], 1500),
        ([("upto", 300), ("pin", 120, 121)], 301),           # pinned token still in window
        ([("upto", 350), ("pin", 100, 350)], 2000),          # the whole window at that time
        ([], 1234),                                          # no promotion
        ([("upto", 600), ("pin", 400, 420), ("upto", 650), ("pin", 600, 640)], 700),
    ]
    _run(cuda_device, 16, 2, lp, w, lcap, plans, seed=701)


def test_pinned_per_unit_schedule(cuda_device):
    """160 sequences (one CTA per unit), each with one promoted range of up to 128 tokens."""
    lp, w, lcap = 64, 128, 64 + 128
    rng = np.random.default_rng(5)
    plans = []
    for b in range(160):
        a = int(rng.integers(lp + 10, 600))
        t0 = int(rng.integers(max(lp, a - w + 1), a + 1))
        t1 = int(min(a + 1, t0 + rng.integers(1, 128)))
        plans.append(([("upto", a), ("pin", t0, t1)], int(a + rng.integers(0, 400))))
    _run(cuda_device, 16, 2, lp, w, lcap, plans, seed=711)


def test_pin_rejects_invalid_ranges(cuda_device):
    """Evicted, out-of-order, future or over-capacity ranges leave the sequence unchanged
    and set PS_DEV_POS_RANGE."""
    dev = cuda_device
    lp, w, lcap = 100, 64, 120
    S, st = _run(dev, 16, 2, lp, w, lcap, [([("upto", 500), ("pin", 450, 460)], 500)], seed=721)
    params = B.make_params(16, 2, D, lp, w, THETA)
    one = lambda v: torch.tensor([v], dtype=torch.int64, device=dev)  # noqa: E731
    before = (S.pin_count.clone(), S.pin_pos.clone(), S.k_pre.clone())
    for t0, t1 in [(430, 440),    # already evicted (t0 <= pos - W)
                   (455, 458),    # not after the last promoted position
                   (490, 502),    # reaches past the latest position
                   (470, 490)]:   # 10 + 20 > capacity 20
        st.zero_()
        B.ps_kv_pin(params, S.full(0, 1), lcap, S.pin_count, S.pin_pos, one(t0), one(t1),
                    one(500), st)
        torch.cuda.synchronize()
        assert st.item() == B.PS_DEV_POS_RANGE, (t0, t1)
        assert torch.equal(S.pin_count, before[0]) and torch.equal(S.pin_pos, before[1])
        assert torch.equal(S.k_pre.isnan(), before[2].isnan())
