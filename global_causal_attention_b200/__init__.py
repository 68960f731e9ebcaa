"""Python binding of the ZGCM-1 attention-core library (libgswa.so, sm_100a).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels behind the C ABI declared in include/gswa.h.  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library is
missing or no sm_100 device is current, the calls raise.

Entry points (same names as the C ABI):
  gswa_fwd       gated sliding-window attention forward  (ZGCM-1 §2.1, Figure 3)
  full_attn_fwd  full causal attention of the global layers (§2.1)
  gswa_bwd, full_attn_bwd, gswa_decode, full_decode  (see include/gswa.h)
  gswa_kv_cache_bytes  KV-cache footprint closed form (§2.3)
  gswa_check_status    read and clear the device status word
  gswa_set_wait_limit_ns  lower the kernels' bounded-wait limit (failure tests)
"""
from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgswa.so")

OK = 0
ERRORS = {
    -1: "INVALID_ARG", -2: "UNSUPPORTED_SHAPE", -3: "MISALIGNED", -4: "WORKSPACE_TOO_SMALL",
    -5: "LAUNCH", -6: "TIMEOUT", -7: "UNIMPLEMENTED", -8: "NO_DEVICE", -9: "SCRATCH_LIMIT",
}
OP_GSWA_FWD, OP_FULL_FWD, OP_GSWA_BWD, OP_FULL_BWD, OP_GSWA_DECODE, OP_FULL_DECODE = range(6)


class GswaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({strerror(code)})")


class Shape(ctypes.Structure):
    """Mirror of gswa_shape_t."""
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("window", ctypes.c_int32),
                ("rope_dims", ctypes.c_int32), ("cache_len", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("eps", ctypes.c_float),
                ("scale", ctypes.c_float)]


_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run global_causal_attention_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I, U = ctypes.c_void_p, ctypes.POINTER(Shape), ctypes.c_int, ctypes.c_size_t
        # (shape, then the pointer arguments, then workspace bytes and the stream)
        sig = {
            "gswa_fwd": [S] + [P] * 9 + [U, P],
            "full_attn_fwd": [S] + [P] * 8 + [U, P],
            "gswa_bwd": [S] + [P] * 16 + [U, P],
            "full_attn_bwd": [S] + [P] * 14 + [U, P],
            "gswa_decode": [S] + [P] * 11 + [U, P],
            "full_decode": [S] + [P] * 10 + [U, P],
            "full_decode_noalloc": [S] + [P] * 10,
            "gswa_qk_prep": [S, I, P, P, P, ctypes.c_int64, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = I
        L._gswa_signatures = sig
        L.gswa_workspace_bytes.argtypes = [I, S]
        L.gswa_workspace_bytes.restype = U
        L.gswa_kv_cache_bytes.argtypes = [I, I, I, I, I, I, ctypes.c_int64]
        L.gswa_kv_cache_bytes.restype = ctypes.c_int64
        L.gswa_check_status.argtypes = [P]
        L.gswa_check_status.restype = I
        L.gswa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.gswa_set_wait_limit_ns.restype = I
        L.gswa_strerror.argtypes = [I]
        L.gswa_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().gswa_strerror(code).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise GswaError(rc, what)


def make_shape(B, T, Hq, Hkv, D=128, window=128, rope_dims=42, rope_base=1e4, eps=1e-6,
               scale=None, cache_len=0) -> Shape:
    return Shape(B, T, Hq, Hkv, D, window, rope_dims, cache_len, rope_base, eps,
                 1.0 / math.sqrt(D) if scale is None else scale)


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(*ts):
    torch = _torch()
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on the GPU")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return torch


def gswa_fwd(q, k, v, g, wq, wk, *, window=128, rope_dims=42, rope_base=1e4, eps=1e-6,
             scale=None, y=None, lse=None, workspace=None, stream=None):
    """Gated SWA forward.  q, g [B,T,Hq,D], k, v [B,T,Hkv,D], wq, wk [D] (bf16, cuda).
    Returns (y [B,T,Hq,D] bf16, lse [B,Hq,T] f32)."""
    torch = _dev(q, k, v, g, wq, wk, y, lse)
    B, T, Hq, D = q.shape
    s = make_shape(B, T, Hq, k.shape[2], D, window, rope_dims, rope_base, eps, scale)
    if y is None:
        y = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    ws, nb = _workspace(OP_GSWA_FWD, s, workspace, q.device)
    _check(lib().gswa_fwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq),
                          _ptr(wk), _ptr(y), _ptr(lse), _ptr(ws), nb, _stream(stream)), "gswa_fwd")
    return y, lse


def full_attn_fwd(q, k, v, wq, wk, *, rope_dims=42, rope_base=1e4, eps=1e-6, scale=None,
                  y=None, lse=None, workspace=None, stream=None):
    """Full causal forward of a global layer (no gate).  Returns (y, lse)."""
    torch = _dev(q, k, v, wq, wk, y, lse)
    B, T, Hq, D = q.shape
    s = make_shape(B, T, Hq, k.shape[2], D, 0, rope_dims, rope_base, eps, scale)
    if y is None:
        y = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    ws, nb = _workspace(OP_FULL_FWD, s, workspace, q.device)
    _check(lib().full_attn_fwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(wq), _ptr(wk),
                               _ptr(y), _ptr(lse), _ptr(ws), nb, _stream(stream)),
           "full_attn_fwd")
    return y, lse


def _bwd_outputs(q, k, gated):
    torch = _torch()
    D = q.shape[-1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(k)
    dg = torch.empty_like(q) if gated else None
    dwq = torch.empty(D, dtype=torch.float32, device=q.device)
    dwk = torch.empty(D, dtype=torch.float32, device=q.device)
    return dq, dk, dv, dg, dwq, dwk


def gswa_bwd(q, k, v, g, wq, wk, y, lse, dy, *, window=128, rope_dims=42, rope_base=1e4, eps=1e-6,
             scale=None, workspace=None, out=None, stream=None):
    """Backward of gswa_fwd given its y and lse and the upstream dy [B,T,Hq,D].
    Returns (dq, dk, dv, dg) bf16 and (dw_q, dw_k) f32, written into `out`
    (a tuple of those six tensors) when given."""
    _dev(q, k, v, g, wq, wk, y, lse, dy, *(out or ()))
    B, T, Hq, D = q.shape
    s = make_shape(B, T, Hq, k.shape[2], D, window, rope_dims, rope_base, eps, scale)
    dq, dk, dv, dg, dwq, dwk = out if out is not None else _bwd_outputs(q, k, True)
    ws, nb = _workspace(OP_GSWA_BWD, s, workspace, q.device)
    _check(lib().gswa_bwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq), _ptr(wk), _ptr(y),
                          _ptr(lse), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dwq), _ptr(dwk),
                          _ptr(ws), nb, _stream(stream)), "gswa_bwd")
    return dq, dk, dv, dg, dwq, dwk


def full_attn_bwd(q, k, v, wq, wk, y, lse, dy, *, rope_dims=42, rope_base=1e4, eps=1e-6, scale=None,
                  workspace=None, out=None, stream=None):
    """Backward of full_attn_fwd.  Returns (dq, dk, dv) bf16 and (dw_q, dw_k) f32,
    written into `out` (those five tensors) when given."""
    _dev(q, k, v, wq, wk, y, lse, dy, *(out or ()))
    B, T, Hq, D = q.shape
    s = make_shape(B, T, Hq, k.shape[2], D, 0, rope_dims, rope_base, eps, scale)
    if out is not None:
        dq, dk, dv, dwq, dwk = out
    else:
        dq, dk, dv, _, dwq, dwk = _bwd_outputs(q, k, False)
    ws, nb = _workspace(OP_FULL_BWD, s, workspace, q.device)
    _check(lib().full_attn_bwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(wq), _ptr(wk), _ptr(y),
                               _ptr(lse), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dwq), _ptr(dwk),
                               _ptr(ws), nb, _stream(stream)), "full_attn_bwd")
    return dq, dk, dv, dwq, dwk


def gswa_qk_prep(x, w, *, rope_dims=42, rope_base=1e4, eps=1e-6, pos0=0, out=None, stream=None):
    """RMSNorm + partial RoPE of x [B, T, H, D] (bf16, cuda) at positions pos0 + t."""
    torch = _dev(x, w, out)
    B, T, H, D = x.shape
    s = make_shape(B, T, H, H, D, 128, rope_dims, rope_base, eps)
    if out is None:
        out = torch.empty_like(x)
    _check(lib().gswa_qk_prep(ctypes.byref(s), H, _ptr(x), _ptr(w), _ptr(out), pos0, _stream(stream)),
           "gswa_qk_prep")
    return out


def gswa_decode(q, k, v, g, wq, wk, k_ring, v_ring, pos, *, rope_dims=42, rope_base=1e4, eps=1e-6,
                scale=None, y=None, stream=None):
    """One gated-SWA decode step over a ring cache [B, Hkv, W, D] (updated in place).
    q, g [B, Hq, D], k, v [B, Hkv, D] bf16; pos [B] int64; returns y [B, Hq, D]."""
    torch = _dev(q, k, v, g, wq, wk, k_ring, v_ring, pos, y)
    B, Hq, D = q.shape
    s = make_shape(B, 1, Hq, k.shape[1], D, k_ring.shape[2], rope_dims, rope_base, eps, scale)
    if y is None:
        y = torch.empty_like(q)
    _check(lib().gswa_decode(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq), _ptr(wk),
                             _ptr(k_ring), _ptr(v_ring), _ptr(pos), _ptr(y), None, 0, _stream(stream)),
           "gswa_decode")
    return y


def full_decode(q, k, v, wq, wk, k_cache, v_cache, pos, *, rope_dims=42, rope_base=1e4, eps=1e-6,
                scale=None, y=None, workspace=None, stream=None):
    """One global-layer decode step over a linear cache [B, Hkv, Tmax, D] (row pos written)."""
    torch = _dev(q, k, v, wq, wk, k_cache, v_cache, pos, y)
    B, Hq, D = q.shape
    s = make_shape(B, 1, Hq, k.shape[1], D, 128, rope_dims, rope_base, eps, scale,
                   cache_len=k_cache.shape[2])
    if y is None:
        y = torch.empty_like(q)
    ws, nb = _workspace(OP_FULL_DECODE, s, workspace, q.device)
    _check(lib().full_decode(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(wq), _ptr(wk),
                             _ptr(k_cache), _ptr(v_cache), _ptr(pos), _ptr(y), _ptr(ws), nb,
                             _stream(stream)), "full_decode")
    return y


def full_decode_noalloc(q, k, v, wq, wk, k_cache, v_cache, pos, y, *, rope_dims=42, rope_base=1e4,
                        eps=1e-6, scale=None, stream=None):
    """full_decode on the library's fixed device scratch: allocates nothing, so
    the output y [B, Hq, D] (bf16, cuda) must be passed in.  Calls that can
    overlap in time share that scratch and must not be issued concurrently."""
    _dev(q, k, v, wq, wk, k_cache, v_cache, pos, y)
    B, Hq, D = q.shape
    s = make_shape(B, 1, Hq, k.shape[1], D, 128, rope_dims, rope_base, eps, scale,
                   cache_len=k_cache.shape[2])
    _check(lib().full_decode_noalloc(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(wq), _ptr(wk),
                                     _ptr(k_cache), _ptr(v_cache), _ptr(pos), _ptr(y), _stream(stream)),
           "full_decode_noalloc")
    return y


def _workspace(op, s, workspace, device):
    torch = _torch()
    need = lib().gswa_workspace_bytes(op, ctypes.byref(s))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace, (workspace.numel() * workspace.element_size() if workspace is not None else 0)


def workspace_bytes(op, shape: Shape) -> int:
    return int(lib().gswa_workspace_bytes(op, ctypes.byref(shape)))


def gswa_kv_cache_bytes(n_global_layers, n_window_layers, window, Hkv, D, bytes_per_elem, T) -> int:
    return int(lib().gswa_kv_cache_bytes(n_global_layers, n_window_layers, window, Hkv, D,
                                         bytes_per_elem, T))


def gswa_check_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib().gswa_check_status(_stream(stream)))


def gswa_set_wait_limit_ns(ns: int) -> None:
    """Make every bounded wait inside the kernels give up after `ns` ns on the
    current device (0 restores the default 4 s); for failure-detection tests."""
    _check(lib().gswa_set_wait_limit_ns(int(ns)), "gswa_set_wait_limit_ns")
