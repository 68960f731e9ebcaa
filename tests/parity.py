"""Element-by-element comparison of a CUDA result with the float64 oracle.

Tolerances (bf16 inputs and outputs, fp32 accumulation):
  forward outputs: max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3;
  gradients:       relative L2 <= 1e-2.  Where the exact gradient is identically
                   zero (a row that sees only its own key has dS = P (dP - D) = 0),
                   the GPU value is the rounding noise of the bf16 y and dA that D
                   and dP are formed from: |dS| <= 2u sum_d |dy sigma v| (u = 2^-9,
                   about 0.08 for N(0,1) inputs), times scale |k~| and the norm's
                   Jacobian, so max |gpu| <= 5e-2 and rms |gpu| <= 5e-3 (an
                   emulation of that rounding gives 2.7e-2 and 1.3e-3).  A wrong
                   mask gives values of order 0.1 and fails.
  weight gradients whose exact value is zero (every row sees only its own
                   key): dw_d is then a sum over all rows of rounding noise
                   projected through the norm's Jacobian, which neither the
                   oracle (exactly 0) nor the per-row outputs bound usefully,
                   so only its finiteness is checked there; the per-row
                   gradients of those cases are still held to the bounds above.
"""
from __future__ import annotations

import numpy as np
import torch

FWD_MAX_ABS = 2e-2
FWD_REL_L2 = 5e-3
GRAD_REL_L2 = 1e-2
GRAD_ZERO_ABS = 5e-2
GRAD_ZERO_RMS = 5e-3


def _np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, np.float64)


def errors(gpu, ref):
    a, b = _np(gpu), _np(ref)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.isfinite(a).all(), "non-finite values in the GPU result"
    d = a - b
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(b), 1e-30)) if d.size else 0.0
    return max_abs, rel


def assert_fwd_close(gpu, ref, what="y"):
    max_abs, rel = errors(gpu, ref)
    assert max_abs <= FWD_MAX_ABS and rel <= FWD_REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def assert_grad_close(gpu, ref, what="grad"):
    """A per-row gradient against the oracle's (relative L2, or the zero-gradient
    noise bounds where the exact gradient is identically zero)."""
    max_abs, rel = errors(gpu, ref)
    if not np.any(_np(ref)):
        rms = float(np.sqrt(np.mean(_np(gpu) ** 2))) if _np(gpu).size else 0.0
        assert max_abs <= GRAD_ZERO_ABS and rms <= GRAD_ZERO_RMS, \
            f"{what}: exact gradient is 0, max_abs={max_abs:.3e} rms={rms:.3e}"
        return max_abs, rel
    assert rel <= GRAD_REL_L2, f"{what}: rel_l2={rel:.3e} (max_abs={max_abs:.3e})"
    return max_abs, rel


def assert_weight_grad_close(dw, ref, what="dw"):
    """A norm-weight gradient dw [D] against the oracle's: relative L2, or only
    finiteness where the exact value is identically zero (module docstring)."""
    if np.any(_np(ref)):
        return assert_grad_close(dw, ref, what)
    a = _np(dw)
    assert np.isfinite(a).all(), f"{what}: non-finite values"
    return float(np.abs(a).max()), 0.0
