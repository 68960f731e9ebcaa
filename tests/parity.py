"""Element-by-element comparison of a CUDA result with the float64 oracle.

Tolerances (bf16 inputs and outputs, fp32 accumulation):
  forward outputs: max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3;
  gradients:       relative L2 <= 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

FWD_MAX_ABS = 2e-2
FWD_REL_L2 = 5e-3
GRAD_REL_L2 = 1e-2


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
    max_abs, rel = errors(gpu, ref)
    assert rel <= GRAD_REL_L2, f"{what}: rel_l2={rel:.3e} (max_abs={max_abs:.3e})"
    return max_abs, rel
