"""Float64 CPU oracle of the ZGCM-1 attention core -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``global_causal_attention_b200``) and never imports it.

The arithmetic lives in ``oracle.c`` (plain loops in float64, each step citing
the page passage it follows); this module only marshals bf16 tensors into
uint16 arrays and float64 outputs back into numpy arrays.

Sources (the pages describe one paper, "ZGCM-1: A Fully Open and Extremely
Efficient Foundation Model for Math and Agentic Search"):
  §2.1 Model overview + Figure 3 caption -- GQA 32/8 heads of dim 128,
      128-token gated SWA, 5 global layers, QK RMSNorm, partial RoPE 0.33,
      GatedSWA(h) = o_proj(A_SWA(q,k,v) ⊙ σ(g_proj(h)));
  §2.3 KV-cache analysis -- 128-token window per SWA layer in the cache;
  §3.2 Mid-training -- RoPE base 10M at 256K.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

_LIB = None

_d = ctypes.c_double
_i = ctypes.c_int
_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def lib(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` selects another build."""
    global _LIB
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _LIB is None:
        _LIB = _bind(ctypes.CDLL(_build.build()))
    return _LIB


def _bind(L):
    L.oracle_qk_prep.argtypes = [_i, _i, _i64, _i, _i, _i, _d, _d, _i64, _p, _p, _p]
    L.oracle_qk_prep.restype = _i
    L.oracle_attn_fwd.argtypes = [_i, _i, _i64, _i, _i, _i, _i, _i, _i, _d, _d, _d,
                                  _p, _p, _p, _p, _p, _p, _i64, _p, _p, _p]
    L.oracle_attn_fwd.restype = _i
    L.oracle_attn_bwd.argtypes = [_i, _i, _i64, _i, _i, _i, _i, _i, _i, _d, _d, _d,
                                  _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]
    L.oracle_attn_bwd.restype = _i
    L.oracle_decode.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _d, _d, _d, _i64, _p,
                                _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]
    L.oracle_decode.restype = _i
    L.oracle_kv_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i64]
    L.oracle_kv_bytes.restype = _i64
    L.oracle_num_threads.argtypes = []
    L.oracle_num_threads.restype = _i
    return L


def _is_f64(t) -> bool:
    return (isinstance(t, np.ndarray) and t.dtype == np.float64) or (
        isinstance(t, torch.Tensor) and t.dtype == torch.float64)


def _arr(t, f64: bool):
    """Input tensor -> contiguous numpy array: bf16 bits (uint16) or float64."""
    if t is None:
        return None
    if f64:
        if isinstance(t, torch.Tensor):
            t = t.detach().to("cpu", torch.float64).numpy()
        return np.ascontiguousarray(t, dtype=np.float64)
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16, t.dtype
        return np.ascontiguousarray(t)
    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a) -> int | None:
    return None if a is None else a.ctypes.data


class _Keep:
    """Holds every converted input array until the C call has returned (a
    pointer to a temporary copy would otherwise dangle)."""

    def __init__(self, f64: bool):
        self.f64 = f64
        self.arrays = []

    def __call__(self, t):
        a = _arr(t, self.f64)
        self.arrays.append(a)
        return _ptr(a)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def num_threads(L=None) -> int:
    return (L or lib()).oracle_num_threads()


def qk_prep(x, w, rope_dims, rope_base, eps, pos0=0, L=None):
    """RMSNorm + partial RoPE of x [B, T, H, D] -> float64 [B, T, H, D].

    Inputs are bf16 tensors, or float64 tensors/arrays (then every input is
    read as float64)."""
    L = L or lib()
    f64 = _is_f64(x)
    keep = _Keep(f64)
    B, T, H, D = x.shape
    out = np.empty((B, T, H, D), np.float64)
    _check(L.oracle_qk_prep(int(f64), B, T, H, D, rope_dims, rope_base, eps, pos0,
                            keep(x), keep(w), _ptr(out)), "qk_prep")
    return out


def attn_fwd(q, k, v, g, wq, wk, *, window, gated, rope_dims, rope_base, eps, scale,
             rows=None, L=None):
    """Forward at all (or the given) query positions.

    Returns (y [B, nrows, Hq, D], lse [B, Hq, nrows]) in float64.
    window <= 0 selects full causal attention; ``gated`` applies σ(g).
    """
    L = L or lib()
    f64 = _is_f64(q)
    keep = _Keep(f64)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    rows_np = None
    nrows = T
    if rows is not None:
        rows_np = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = rows_np.shape[0]
    y = np.empty((B, nrows, Hq, D), np.float64)
    lse = np.empty((B, Hq, nrows), np.float64)
    _check(L.oracle_attn_fwd(int(f64), B, T, Hq, Hkv, D, window, int(bool(gated)), rope_dims,
                             rope_base, eps, scale, keep(q), keep(k), keep(v),
                             keep(g) if gated else None, keep(wq), keep(wk), nrows, _ptr(rows_np),
                             _ptr(y), _ptr(lse)), "attn_fwd")
    return y, lse


def attn_bwd(q, k, v, g, wq, wk, dy, *, window, gated, rope_dims, rope_base, eps, scale,
             L=None):
    """Gradients (dq, dk, dv, dg or None, dwq, dwk) in float64."""
    L = L or lib()
    f64 = _is_f64(q)
    keep = _Keep(f64)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dq = np.empty((B, T, Hq, D), np.float64)
    dk = np.empty((B, T, Hkv, D), np.float64)
    dv = np.empty((B, T, Hkv, D), np.float64)
    dg = np.empty((B, T, Hq, D), np.float64) if gated else None
    dwq = np.empty(D, np.float64)
    dwk = np.empty(D, np.float64)
    _check(L.oracle_attn_bwd(int(f64), B, T, Hq, Hkv, D, window, int(bool(gated)), rope_dims,
                             rope_base, eps, scale, keep(q), keep(k), keep(v),
                             keep(g) if gated else None, keep(wq), keep(wk), keep(dy), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dwq), _ptr(dwk)), "attn_bwd")
    return dq, dk, dv, dg, dwq, dwk


def decode(q, k, v, g, wq, wk, k_cache, v_cache, pos, *, window, gated, rope_dims,
           rope_base, eps, scale, L=None):
    """One decode step.  window > 0: ring cache [B, Hkv, W, D]; else linear
    cache [B, Hkv, Tmax, D].  Returns (y [B, Hq, D], k_new_prepared [B, Hkv, D])."""
    L = L or lib()
    f64 = _is_f64(q)
    keep = _Keep(f64)
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    Tmax = k_cache.shape[2]
    pos_np = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(B))
    y = np.empty((B, Hq, D), np.float64)
    kp = np.empty((B, Hkv, D), np.float64)
    _check(L.oracle_decode(int(f64), B, Hq, Hkv, D, window, int(bool(gated)), rope_dims,
                           rope_base, eps, scale, Tmax, _ptr(pos_np), keep(q), keep(k),
                           keep(v), keep(g) if gated else None, keep(wq), keep(wk),
                           keep(k_cache), keep(v_cache), _ptr(y), _ptr(kp)), "decode")
    return y, kp


def kv_bytes(n_global, n_window, window, Hkv, D, bytes_per_elem, T, L=None) -> int:
    """KV-cache bytes of a stack at context length T (§2.3 closed form)."""
    L = L or lib()
    return int(L.oracle_kv_bytes(n_global, n_window, window, Hkv, D, bytes_per_elem, T))


def shape_kwargs(s) -> dict:
    """Keyword arguments of the oracle calls for a ``workloads.Shape``."""
    return dict(rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
