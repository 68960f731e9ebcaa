"""Dense float64 restatement of the attention core from library routines.

Used only to pin the oracle: the norm is ``torch.nn.functional.rms_norm``, the
rotation is the textbook complex-exponential form of RoPE (RoFormer:
(x_p + i x_{p+R/2}) * exp(i * pos * base^(-2p/R))), the attention is
``scaled_dot_product_attention`` with a dense boolean band mask and
``enable_gqa`` (query head h reads KV head h // (Hq/Hkv)), the gate is
``torch.sigmoid`` and every gradient comes from autograd.  None of this shares
code with the oracle's loops, so a wrong sign, index or dropped term on either
side shows up as a mismatch.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F

f64 = torch.float64


def rope_complex(u: torch.Tensor, pos: torch.Tensor, R: int, base: float) -> torch.Tensor:
    """Rotate the first R dims of u [..., T, H, D] as complex pairs (p, p + R/2)."""
    if R == 0:
        return u
    half = R // 2
    theta = torch.pow(torch.tensor(base, dtype=f64), -2.0 * torch.arange(half, dtype=f64) / R)
    rot = torch.polar(torch.ones_like(theta)[None, :].expand(pos.numel(), half),
                      pos.to(f64)[:, None] * theta[None, :])          # [T, half]
    z = torch.complex(u[..., :half], u[..., half:R]) * rot[:, None, :]
    return torch.cat([z.real, z.imag, u[..., R:]], dim=-1)


def prep(x, w, R, base, eps, pos):
    return rope_complex(F.rms_norm(x, (x.shape[-1],), weight=w, eps=eps), pos, R, base)


def band_mask(T: int, window: int) -> torch.Tensor:
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    m = j <= i
    if window > 0:
        m = m & (j > i - window)
    return m


def forward(q, k, v, g, wq, wk, *, window, gated, rope_dims, rope_base, eps, scale):
    """y [B,T,Hq,D] and lse [B,Hq,T] for float64 inputs."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    pos = torch.arange(T, dtype=f64)
    qt = prep(q, wq, rope_dims, rope_base, eps, pos).transpose(1, 2)   # [B,Hq,T,D]
    kt = prep(k, wk, rope_dims, rope_base, eps, pos).transpose(1, 2)   # [B,Hkv,T,D]
    vt = v.transpose(1, 2)
    m = band_mask(T, window)
    A = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale,
                                       enable_gqa=True).transpose(1, 2)
    y = A * torch.sigmoid(g) if gated else A
    s = scale * qt @ kt.repeat_interleave(Hq // Hkv, dim=1).transpose(-1, -2)
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return y, lse


def gradients(q, k, v, g, wq, wk, dy, *, window, gated, **kw):
    """Autograd gradients of sum(y * dy) w.r.t. every input (float64)."""
    leaves = [t.detach().clone().requires_grad_(True) for t in (q, k, v, g, wq, wk)]
    y, _ = forward(*leaves, window=window, gated=gated, **kw)
    (y * dy).sum().backward()
    return [t.grad for t in leaves]
