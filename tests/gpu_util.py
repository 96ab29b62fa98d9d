"""Shared helpers of the GPU parity tests (comparison metrics; no attention arithmetic)."""
import numpy as np
import torch

# Float tolerance of the parity bar: bf16 inputs, fp32 accumulation.
MAX_ABS = 2e-2
REL_RMS = 5e-3


def f64(t) -> np.ndarray:
    """Exact bf16/fp32 -> float64 numpy copy of a torch tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def errors(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    d = got - want
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_close(got, want, what="", max_abs=MAX_ABS, rel_rms=REL_RMS):
    got = np.asarray(got, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    m, r = errors(got, want)
    assert m <= max_abs and r <= rel_rms, f"{what}: max_abs={m:.3e} rel_rms={r:.3e}"
    return m, r


# Margin of the backward's element bar over the error of its rounding model: the model
# (tests/bwd_model.py) keeps every fp32 step exact, while the kernel adds fp32 accumulation
# order and the fp32 exponential; more importantly, two runs of the same bf16 rounding points
# on slightly different fp32 values give different largest errors over a tensor.
GRAD_MODEL_MARGIN = 1.25


def assert_close_grad(got, want, what="", tol=MAX_ABS, rel_rms=REL_RMS, model_err=0.0):
    """Bar for the backward's bf16 gradients: per element |got - want| <= bar * max(1, r) with
    r the rms of the reference over that row's last axis (the 128 head dims), and
    rel_rms <= 5e-3 per tensor.  bar = max(2e-2, GRAD_MODEL_MARGIN * model_err), where
    model_err is the same element measure of the rounding model (tests/bwd_model.py: the
    kernels' bf16 points for P, O, dS and the outputs) on the same inputs.  The kernel rounds
    P and dS to bf16 before the products, so an element's error scales with the magnitude of
    the terms its sum shares with the rest of the row (a prefix key's dK sums every query's
    contribution), not with the element itself; and gradients exceed 1, where one bf16 step
    is larger than an absolute 2e-2.  A wrong or missing row still misses by about the row's
    own rms."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    m, r = errors(got, want)
    row = np.sqrt((want ** 2).mean(axis=-1, keepdims=True)) if want.size else want
    scaled = float((np.abs(got - want) / np.maximum(1.0, row)).max()) if got.size else 0.0
    bar = max(tol, GRAD_MODEL_MARGIN * model_err)
    print(f"{what}: max_abs={m:.3e} scaled={scaled:.3e} model={model_err:.3e} bar={bar:.3e} "
          f"rel_rms={r:.3e} max|ref|={float(np.abs(want).max()) if want.size else 0.0:.3f}")
    assert scaled <= bar and r <= rel_rms, \
        f"{what}: max_abs={m:.3e} scaled={scaled:.3e} bar={bar:.3e} rel_rms={r:.3e}"
    return scaled, r
