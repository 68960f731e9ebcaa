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
                   mask gives values of order 0.1 and fails.  For a sum over n
                   rows of such noise (the weight gradients) both bounds grow
                   with sqrt(n), the random-walk growth of independent errors.
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


def assert_grad_close(gpu, ref, what="grad", terms=1):
    """`terms`: rows summed into each element (1 for per-row gradients)."""
    max_abs, rel = errors(gpu, ref)
    if not np.any(_np(ref)):
        rms = float(np.sqrt(np.mean(_np(gpu) ** 2))) if _np(gpu).size else 0.0
        grow = float(np.sqrt(max(terms, 1)))
        assert max_abs <= GRAD_ZERO_ABS * grow and rms <= GRAD_ZERO_RMS * grow, \
            f"{what}: exact gradient is 0, max_abs={max_abs:.3e} rms={rms:.3e}"
        return max_abs, rel
    assert rel <= GRAD_REL_L2, f"{what}: rel_l2={rel:.3e} (max_abs={max_abs:.3e})"
    return max_abs, rel
