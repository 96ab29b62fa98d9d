"""GPU parity of the masked prefill backward (dQ, dK, dV) against the float64 oracle.

The forward runs first through the C ABI (its bf16 output and fp32 lse are what a trainer
keeps); the backward then gets dO.  Every row of dQ and every key row of dK, dV is checked
on small shapes (ragged tails, W = 1, no prefix, dense causal, prefix longer than a tile,
GQA groups 2, 7 and 8); at the full truncated-backprop size, sampled rows and keys.
Bar: |got - ref| <= bar * max(1, rms of the reference row) per element and rel_rms <= 5e-3
per tensor, with bar = max(2e-2, 1.25 x the same measure of the rounding model of the
kernels (tests/bwd_model.py) on the same inputs).  P and dS are rounded to bf16 before the
products, so an element's error scales with its row's terms; gradients exceed 1, where a
bf16 step is larger than 2e-2; at a softmax scale above the default, peakier P makes dS
larger and the model's error exceeds 2e-2 by itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from tests import bwd_model as M
from tests.gpu_util import assert_close_grad, f64

pytestmark = pytest.mark.gpu

D = 128


def _forward_backward(dev, Bn, S, hq, hkv, lp, w, seed, scale=0.0):
    params = B.make_params(hq, hkv, D, lp, w, softmax_scale=scale)
    q = synth.normal_bf16((Bn, S, hq, D), seed, dev)
    k = synth.normal_bf16((Bn, S, hkv, D), seed + 1, dev)
    v = synth.normal_bf16((Bn, S, hkv, D), seed + 2, dev)
    do = synth.normal_bf16((Bn, S, hq, D), seed + 3, dev)
    out = torch.empty((Bn, S, hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Bn, hq, S), dtype=torch.float32, device=dev)
    ws = torch.empty(B.ps_prefill_workspace_bytes(params, Bn, S), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    B.ps_masked_prefill_attn(params, q, k, v, Bn, S, out, lse, None, ws, st)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    wsb = torch.empty(B.ps_prefill_bwd_workspace_bytes(params, Bn, S), dtype=torch.uint8,
                      device=dev)
    B.ps_masked_prefill_attn_bwd(params, q, k, v, out, do, lse, Bn, S, dq, dk, dv, wsb, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    return params, (q, k, v, do), (dq, dk, dv), (out, lse, wsb, st)


def _check_all(inputs, grads, lp, w, scale):
    q, k, v, do = (f64(t) for t in inputs)
    dq, dk, dv = (f64(t) for t in grads)
    for b in range(q.shape[0]):
        wq, wk, wv = O.prefill_backward_reference(q[b], k[b], v[b], do[b], lp, w, scale)
        _, mq, mk, mv = M.forward_backward(q[b], k[b], v[b], do[b], lp, w, scale)
        assert_close_grad(dq[b], wq, f"dq b={b}", model_err=M.scaled_error(mq, wq))
        assert_close_grad(dk[b], wk, f"dk b={b}", model_err=M.scaled_error(mk, wk))
        assert_close_grad(dv[b], wv, f"dv b={b}", model_err=M.scaled_error(mv, wv))


@pytest.mark.parametrize("S,lp,w,hq,hkv", [(520, 16, 200, 4, 2), (300, 0, 64, 4, 2),
                                          (128, 5, 1, 4, 2), (1, 0, 1, 4, 2),
                                          (129, 40, 1000, 4, 2), (640, 130, 130, 4, 2),
                                          (384, 100, 128, 16, 2)])
def test_prefill_bwd_every_row_and_key(cuda_device, S, lp, w, hq, hkv):
    _, inputs, grads, _ = _forward_backward(cuda_device, 2, S, hq, hkv, lp, w, seed=300 + S)
    _check_all(inputs, grads, lp, w, 1 / math.sqrt(D))


def test_prefill_bwd_group_seven_custom_scale(cuda_device):
    _, inputs, grads, _ = _forward_backward(cuda_device, 1, 300, 28, 4, 20, 100, seed=31,
                                            scale=0.3)
    _check_all(inputs, grads, 20, 100, 0.3)


def test_prefill_bwd_deterministic_and_closed_form_sums(cuda_device):
    """dK/dV are reduced inside one CTA (no atomics): a second call is bit-identical.  The
    softmax rows sum to one, so sum_j dV_j equals the group's sum of dO (closed form)."""
    params, inputs, grads, (out, lse, wsb, st) = _forward_backward(cuda_device, 2, 700, 8, 2,
                                                                   64, 256, seed=55)
    q, k, v, do = inputs
    again = [torch.empty_like(t) for t in grads]
    B.ps_masked_prefill_attn_bwd(params, q, k, v, out, do, lse, 2, 700, *again, wsb, st)
    torch.cuda.synchronize()
    for g, a in zip(grads, again):
        assert torch.equal(g, a)
    dv = f64(grads[2])
    want = f64(do).reshape(2, 700, 2, 4, D).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), want, rtol=0, atol=0.5)


def test_prefill_bwd_truncated_context_full_size(cuda_device):
    """Full truncated-backprop shape: batch 4, 8192 tokens = 4 x W with W = 2048,
    L_prefix = 256, 28 query / 4 KV heads.  Sampled dQ rows and dK/dV keys (prefix ends,
    window edges, tail) of one batch element and one KV-head group (its 7 query heads)."""
    wl = synth.WORKLOADS["prefill_b4_s8192_w2048"]
    _, inputs, grads, _ = _forward_backward(cuda_device, wl.batch, wl.seq, wl.n_q_heads,
                                            wl.n_kv_heads, wl.l_prefix, wl.window,
                                            seed=synth.seed_for(3, 5))
    for t in grads:
        assert torch.isfinite(t.float()).all()
    b, kvh = 3, 1
    g = wl.n_q_heads // wl.n_kv_heads
    hs = slice(kvh * g, (kvh + 1) * g)
    q, k, v, do = (t[b] for t in inputs)
    qf, dof = f64(q[:, hs]), f64(do[:, hs])
    kf, vf = f64(k[:, kvh:kvh + 1]), f64(v[:, kvh:kvh + 1])
    rows = [0, 127, 255, 256, 2303, 2304, 4096, 6143, 8191]
    keys = [0, 200, 255, 256, 1000, 4095, 6144, 8190, 8191]
    wq, wk, wv = O.prefill_backward_reference(qf, kf, vf, dof, wl.l_prefix, wl.window,
                                              1 / math.sqrt(D), rows=rows, keys=keys)
    dq, dk, dv = grads
    assert_close_grad(f64(dq[b][rows][:, hs]), wq, "dq rows")
    assert_close_grad(f64(dk[b][keys][:, kvh:kvh + 1]), wk, "dk keys")
    assert_close_grad(f64(dv[b][keys][:, kvh:kvh + 1]), wv, "dv keys")


def test_prefill_bwd_passes_bit_identical(cuda_device):
    """A workspace smaller than the whole batch needs runs the batch in passes of as many
    sequences as it holds (one, two, then all three here); every pass covers whole sequences,
    so the gradients are bit-identical to the one-pass call.  One of the batch-3 sequences is
    also checked against the oracle."""
    S, hq, hkv, lp, w = 390, 8, 2, 50, 128
    params, inputs, grads, (out, lse, wsb, st) = _forward_backward(cuda_device, 3, S, hq, hkv,
                                                                   lp, w, seed=77)
    q, k, v, do = inputs
    sizes = [B.ps_prefill_bwd_workspace_bytes(params, n, S) for n in (1, 2, 3)]
    assert sizes[0] < sizes[1] < sizes[2] == wsb.numel()
    for nbytes in sizes[:2] + [sizes[1] + 1000]:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=cuda_device)
        again = [torch.full_like(t, float("nan")) for t in grads]
        B.ps_masked_prefill_attn_bwd(params, q, k, v, out, do, lse, 3, S, *again, ws, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        for g, a in zip(grads, again):
            assert torch.equal(g.view(torch.int16), a.view(torch.int16))
    _check_all([t[2:3] for t in inputs], [t[2:3] for t in grads], lp, w, 1 / math.sqrt(D))
