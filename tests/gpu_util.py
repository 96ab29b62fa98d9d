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
