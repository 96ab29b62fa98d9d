"""A CPU model of where the masked prefill and its backward round (test infrastructure only).

This is NOT the oracle: the oracle (``oracle/``) computes the gradients exactly, in float64.
This module repeats the same chain rule with the bf16 roundings the CUDA kernels apply, so
that a GPU test can compare the kernel's error against the error those roundings alone
produce, and so that the bar of the backward's parity tests rests on a committed model.

Rounding points modelled (everything else is float64, since fp32 accumulation and the fp32
exponential add errors some 2^13 times smaller than a bf16 rounding):

forward (masked prefill, tcgen05 kernel):
  * the probabilities p_ij = exp(s_ij - m_i) enter the P.V product as bf16;
  * the row sum l_i adds the unrounded p_ij;
  * O_i = (sum_j bf16(p_ij) V_j) / l_i is stored as bf16; lse_i is fp32 (kept exact here).
backward (dK/dV kernel, then the dQ GEMM):
  * P_ij = exp(s_ij - lse_i) from the forward's lse;
  * D_i = <dO_i, O_i> with the forward's bf16 O;
  * dV_j = sum_i bf16(P_ij) dO_i;
  * dS_ij = P_ij (dP_ij - D_i), stored as bf16 and used as bf16 by both dK and dQ;
  * dK_j = scale sum_i bf16(dS_ij) Q_i, dQ_i = scale sum_j bf16(dS_ij) K_j;
  * dQ, dK, dV stored as bf16.

With ``exact=True`` no rounding is applied, and the result must equal the oracle's
(``tests/test_bwd_model.py`` checks this, which pins the model's algebra).
"""
from __future__ import annotations

import numpy as np
import torch


def bf16(x: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (nearest even), returned as float64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def _mask(S: int, l_prefix: int, window: int) -> np.ndarray:
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    return (j <= i) & ((j < l_prefix) | (j > i - window))


def forward_backward(Q, K, V, dO, l_prefix: int, window: int, scale: float,
                     exact: bool = False):
    """Model of the kernels' forward output and gradients for one sequence.

    Q, dO: [S, Hq, D]; K, V: [S, Hkv, D] (bf16-exact values as float64).
    Returns (O [S, Hq, D], dQ [S, Hq, D], dK [S, Hkv, D], dV [S, Hkv, D]).
    """
    r = (lambda x: x) if exact else bf16
    Q, K, V, dO = (np.asarray(t, np.float64) for t in (Q, K, V, dO))
    S, hq, d = Q.shape
    hkv = K.shape[1]
    g = hq // hkv
    vis = _mask(S, l_prefix, window)
    O = np.zeros_like(Q)
    dQ = np.zeros_like(Q)
    dK = np.zeros((S, hkv, d))
    dV = np.zeros((S, hkv, d))
    for h in range(hq):
        kv = h // g
        s = np.where(vis, (Q[:, h] @ K[:, kv].T) * scale, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        lsum = p.sum(axis=1, keepdims=True)
        O[:, h] = r((r(p) @ V[:, kv]) / lsum)
        lse = m + np.log(lsum)
        # backward: P from the forward's lse, D from its bf16 output
        P = np.exp(s - lse)
        dP = dO[:, h] @ V[:, kv].T
        Dr = (dO[:, h] * O[:, h]).sum(axis=1, keepdims=True)
        dS = r(P * (dP - Dr))
        dV[:, kv] += r(P).T @ dO[:, h]
        dK[:, kv] += dS.T @ Q[:, h]
        dQ[:, h] = r(scale * (dS @ K[:, kv]))
    return O, dQ, r(scale * dK), r(dV)


def scaled_error(got: np.ndarray, want: np.ndarray) -> float:
    """max over elements of |got - want| / max(1, rms of the reference row over its last
    axis): the element measure of the backward's parity bar."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    if want.size == 0:
        return 0.0
    row = np.sqrt((want ** 2).mean(axis=-1, keepdims=True))
    return float((np.abs(got - want) / np.maximum(1.0, row)).max())
