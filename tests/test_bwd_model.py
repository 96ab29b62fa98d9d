"""Pins of the backward's rounding model (tests/bwd_model.py), CPU only.

The model is the oracle's chain rule with the kernels' bf16 rounding points added; the GPU
parity tests of the backward take their element bar from it.  Here: with rounding switched
off it must reproduce the oracle exactly (so its algebra is the oracle's, not a copy of the
kernel's), and with rounding on, at the default softmax scale, it stays inside the plain
floating-point bar (|err| <= 2e-2 per element, relative to max(1, row rms); rel_rms <= 5e-3).
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from tests import bwd_model as M

D = 128


def _inputs(S, hq, hkv, seed):
    return (synth.normal_bf16((S, hq, D), seed).double().numpy(),
            synth.normal_bf16((S, hkv, D), seed + 1).double().numpy(),
            synth.normal_bf16((S, hkv, D), seed + 2).double().numpy(),
            synth.normal_bf16((S, hq, D), seed + 3).double().numpy())


@pytest.mark.parametrize("S,lp,w,hq,hkv,scale", [(200, 16, 70, 4, 2, None), (128, 5, 1, 4, 2, None),
                                                (150, 0, 64, 4, 2, None), (160, 20, 100, 28, 4, 0.3)])
def test_exact_model_is_the_oracle(S, lp, w, hq, hkv, scale):
    scale = scale or 1 / math.sqrt(D)
    q, k, v, do = _inputs(S, hq, hkv, 11 + S)
    o, dq, dk, dv = M.forward_backward(q, k, v, do, lp, w, scale, exact=True)
    wo, _ = O.prefill_reference(q, k, v, lp, w, scale)
    wq, wk, wv = O.prefill_backward_reference(q, k, v, do, lp, w, scale)
    for got, want in ((o, wo), (dq, wq), (dk, wk), (dv, wv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)


@pytest.mark.parametrize("S,lp,w,hq,hkv", [(520, 16, 200, 4, 2), (300, 0, 64, 4, 2),
                                          (384, 100, 128, 16, 2)])
def test_rounded_model_inside_plain_bar_at_default_scale(S, lp, w, hq, hkv):
    scale = 1 / math.sqrt(D)
    q, k, v, do = _inputs(S, hq, hkv, 31 + S)
    _, dq, dk, dv = M.forward_backward(q, k, v, do, lp, w, scale)
    wq, wk, wv = O.prefill_backward_reference(q, k, v, do, lp, w, scale)
    for got, want in ((dq, wq), (dk, wk), (dv, wv)):
        assert 0 < M.scaled_error(got, want) <= 2e-2
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3


def test_rounded_model_differs_from_exact():
    """Each modelled rounding moves the result (a model that rounded nothing would give a
    zero bar)."""
    q, k, v, do = _inputs(130, 4, 2, 7)
    ex = M.forward_backward(q, k, v, do, 10, 50, 0.1, exact=True)
    rd = M.forward_backward(q, k, v, do, 10, 50, 0.1)
    for a, b in zip(ex, rd):
        assert np.abs(a - b).max() > 0
