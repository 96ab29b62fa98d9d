"""GPU parity of the masked prefill (two-level filtered, tcgen05) against the oracle.

The tile plan the kernel ran must equal the oracle's brute-force plan bit for bit; outputs
must hold max_abs <= 2e-2 and rel_rms <= 5e-3 (and lse within 2e-2) row by row.
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


def _run(dev, Bn, S, hq, hkv, lp, w, seed, want_plan=True, scale=0.0):
    params = B.make_params(hq, hkv, D, lp, w, softmax_scale=scale)
    q = synth.normal_bf16((Bn, S, hq, D), seed, dev)
    k = synth.normal_bf16((Bn, S, hkv, D), seed + 1, dev)
    v = synth.normal_bf16((Bn, S, hkv, D), seed + 2, dev)
    out = torch.full((Bn, S, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((Bn, hq, S), float("nan"), dtype=torch.float32, device=dev)
    n = B.ps_prefill_plan_tiles(params, S)
    plan = torch.full((n, 3), -1, dtype=torch.int32, device=dev) if want_plan else None
    ws = torch.empty(B.ps_prefill_workspace_bytes(params, Bn, S), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    got_n = B.ps_masked_prefill_attn(params, q, k, v, Bn, S, out, lse, plan, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    assert got_n == n
    return q, k, v, out, lse, plan


def _check_rows(q, k, v, out, lse, lp, w, rows, scale=None, heads=None):
    Bn, S, hq, _ = q.shape
    scale = scale or 1 / math.sqrt(D)
    qf, kf, vf, of, lf = f64(q), f64(k), f64(v), f64(out), f64(lse)
    for b in range(Bn):
        want, want_lse = O.prefill_reference(qf[b], kf[b], vf[b], lp, w, scale, rows=rows)
        got = of[b, rows]
        if heads is not None:
            want, got = want[:, heads], got[:, heads]
            want_lse = want_lse[:, heads]
        assert_close(got, want, f"b={b}")
        gl = lf[b][:, rows].T if heads is None else lf[b][heads][:, rows].T
        assert np.abs(gl - want_lse).max() < 2e-2


@pytest.mark.parametrize("S,lp,w", [(520, 16, 200), (300, 0, 64), (128, 5, 1), (1, 0, 1),
                                   (129, 40, 1000), (640, 130, 130)])
def test_prefill_plan_bit_exact_and_all_rows(cuda_device, S, lp, w):
    q, k, v, out, lse, plan = _run(cuda_device, 2, S, 4, 2, lp, w, seed=100 + S)
    want_plan = O.tile_plan(S, lp, w, 128, 128)
    np.testing.assert_array_equal(plan.cpu().numpy(), want_plan)
    _check_rows(q, k, v, out, lse, lp, w, list(range(S)))


def test_prefill_dense_causal_when_window_covers_sequence(cuda_device):
    S = 384
    q, k, v, out, lse, plan = _run(cuda_device, 1, S, 8, 1, 0, S, seed=7)
    p = plan.cpu().numpy()
    assert (p[p[:, 0] == p[:, 1]][:, 2] == B.PS_TILE_PARTIAL).all()
    assert (p[p[:, 0] != p[:, 1]][:, 2] == B.PS_TILE_FULL).all()
    _check_rows(q, k, v, out, lse, 0, S, list(range(S)))


def test_prefill_custom_scale_group_seven(cuda_device):
    q, k, v, out, lse, _ = _run(cuda_device, 1, 300, 28, 4, 20, 100, seed=9, scale=0.3)
    _check_rows(q, k, v, out, lse, 20, 100, list(range(0, 300, 7)), scale=0.3)


def test_prefill_truncated_context_full_size(cuda_device):
    """Truncated-backprop context forward at full size: batch 4, 8192 tokens = 4 x W with
    W = 2048, L_prefix = 256, 28 query / 4 KV heads.  Full plan bit-exact; sampled rows
    (prefix, warm-up, window edges, tail) checked against the oracle for every head."""
    wl = synth.WORKLOADS["prefill_b4_s8192_w2048"]
    q, k, v, out, lse, plan = _run(cuda_device, wl.batch, wl.seq, wl.n_q_heads, wl.n_kv_heads,
                                   wl.l_prefix, wl.window, seed=synth.seed_for(3))
    want_plan = O.tile_plan(wl.seq, wl.l_prefix, wl.window, 128, 128)
    np.testing.assert_array_equal(plan.cpu().numpy(), want_plan)
    flags = want_plan[:, 2]
    assert ((flags == O.TILE_FULL).sum(), (flags == O.TILE_PARTIAL).sum()) == (935, 110)
    rows = [0, 1, 127, 128, 255, 256, 257, 2047, 2303, 2304, 2305, 4095, 4096, 5000, 6143, 6144,
            8000, 8190, 8191]
    _check_rows(q, k, v, out, lse, wl.l_prefix, wl.window, rows)
    assert torch.isfinite(out.float()).all()
