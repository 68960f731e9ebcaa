"""The layer stack of ZGCM-1's attention core, driven through the C ABI.

ZGCM-1 §2.1 Model overview: 32 decoder layers; layers 6, 12, 18, 24 and 30
(1-based) are global layers (full causal attention over the whole context, no
gate), the other 27 are gated sliding-window layers (window 128).  The
Figure 3 caption puts the last global layer at layer 29 counted from 0, so
layers 31 and 32 are sliding-window layers.  §2.2 (hybrid-attention
experiments) compares the same backbone with 1:1, 3:1 and 5:1 ratios of
sliding-window to global layers; `global_layers` gives each schedule.

This module is control flow only: every layer is one call of an entry point
of libgswa.so (gswa_fwd / full_attn_fwd for a prefill, gswa_decode /
full_decode for a decode step), on the caller's stream, in layer order.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (OP_FULL_DECODE, OP_FULL_FWD, OP_GSWA_FWD, full_attn_fwd, full_decode, gswa_decode,
               gswa_fwd, make_shape, workspace_bytes)


def global_layers(n_layers: int = 32, swa_per_global: int = 5) -> tuple:
    """1-based indices of the global layers of an r:1 schedule (r sliding-window
    layers per global layer): every (r + 1)-th layer.  32 layers at 5:1 give
    (6, 12, 18, 24, 30)."""
    if n_layers < 0 or swa_per_global < 0:
        raise ValueError("n_layers and swa_per_global must be >= 0")
    return tuple(l for l in range(1, n_layers + 1) if l % (swa_per_global + 1) == 0)


@dataclass
class AttentionStack:
    """Schedule and attention settings of a stack of `n_layers` layers."""
    n_layers: int = 32
    swa_per_global: int = 5
    window: int = 128
    rope_dims: int = 42
    rope_base: float = 1e4
    eps: float = 1e-6
    scale: float | None = None

    def __post_init__(self):
        self.globals = frozenset(global_layers(self.n_layers, self.swa_per_global))

    def is_global(self, layer: int) -> bool:
        """Layer `layer` (1-based) is a global (full causal) layer."""
        return layer in self.globals

    def kinds(self):
        return ["global" if self.is_global(l) else "swa" for l in range(1, self.n_layers + 1)]

    def _kw(self):
        return dict(rope_dims=self.rope_dims, rope_base=self.rope_base, eps=self.eps, scale=self.scale)

    @staticmethod
    def _per_layer(x, n, what):
        """A per-layer sequence of length n, or one value used by every layer."""
        if isinstance(x, (list, tuple)):
            if len(x) != n:
                raise ValueError(f"{what}: {len(x)} entries for {n} layers")
            return list(x)
        return [x] * n

    # ------------------------------------------------------------------ prefill
    def prefill_workspace(self, B, T, Hq, Hkv, device):
        """One workspace big enough for either kind of layer at this shape."""
        import torch
        s_swa = make_shape(B, T, Hq, Hkv, 128, self.window, **self._kw())
        s_full = make_shape(B, T, Hq, Hkv, 128, 0, **self._kw())
        n = max(workspace_bytes(OP_GSWA_FWD, s_swa), workspace_bytes(OP_FULL_FWD, s_full), 1)
        return torch.empty(n, dtype=torch.uint8, device=device)

    def prefill_calls(self, inputs, outputs, workspace=None, stream=None):
        """The stack's prefill as a list of (entry point, callable), one per
        layer in order.  inputs: per layer a dict with q, k, v, g, wq, wk (g is
        unused by global layers), or one dict for every layer.  outputs: per
        layer a (y, lse) pair of buffers (y [B,T,Hq,D] bf16, lse [B,Hq,T] f32),
        or one pair for every layer."""
        ins = self._per_layer(inputs, self.n_layers, "inputs")
        outs = self._per_layer(outputs, self.n_layers, "outputs")
        if workspace is None:
            q = ins[0]["q"]
            B, T, Hq, _ = q.shape
            workspace = self.prefill_workspace(B, T, Hq, ins[0]["k"].shape[2], q.device)
        kw = self._kw()
        calls = []
        for l in range(1, self.n_layers + 1):
            x, (y, lse) = ins[l - 1], outs[l - 1]
            if self.is_global(l):
                calls.append(("full_attn_fwd", lambda x=x, y=y, lse=lse: full_attn_fwd(
                    x["q"], x["k"], x["v"], x["wq"], x["wk"], y=y, lse=lse, workspace=workspace,
                    stream=stream, **kw)))
            else:
                calls.append(("gswa_fwd", lambda x=x, y=y, lse=lse: gswa_fwd(
                    x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=self.window, y=y, lse=lse,
                    workspace=workspace, stream=stream, **kw)))
        return calls

    def prefill(self, inputs, outputs, workspace=None, stream=None):
        """Run every layer's forward in order (asynchronously on `stream`)."""
        for _, fn in self.prefill_calls(inputs, outputs, workspace, stream):
            fn()
        return outputs

    # ------------------------------------------------------------------- decode
    def decode_workspace(self, B, Hq, Hkv, cache_len, device):
        import torch
        s = make_shape(B, 1, Hq, Hkv, 128, self.window, cache_len=cache_len, **self._kw())
        return torch.empty(max(workspace_bytes(OP_FULL_DECODE, s), 1), dtype=torch.uint8, device=device)

    def decode_calls(self, inputs, caches, pos, outputs, workspace=None, stream=None):
        """One decode step of the stack as (entry point, callable) pairs.
        inputs: per layer a dict with the new token's q, g [B,Hq,D], k, v
        [B,Hkv,D] and wq, wk (or one dict for every layer); caches: per layer
        a (k_cache, v_cache) pair -- a ring [B,Hkv,window,D] for a
        sliding-window layer, a linear cache [B,Hkv,Tmax,D] for a global layer
        (or one pair per kind: {"swa": ..., "global": ...}); pos [B] int64
        (device); outputs: per layer a y [B,Hq,D] buffer, or one for all."""
        ins = self._per_layer(inputs, self.n_layers, "inputs")
        outs = self._per_layer(outputs, self.n_layers, "outputs")
        if isinstance(caches, dict):
            cs = [caches["global" if self.is_global(l) else "swa"] for l in range(1, self.n_layers + 1)]
        else:
            cs = self._per_layer(caches, self.n_layers, "caches")
        if workspace is None:
            lin = next((cs[l - 1] for l in range(1, self.n_layers + 1) if self.is_global(l)), None)
            if lin is not None:
                q = ins[0]["q"]
                workspace = self.decode_workspace(q.shape[0], q.shape[1], ins[0]["k"].shape[1],
                                                  lin[0].shape[2], q.device)
        kw = self._kw()
        calls = []
        for l in range(1, self.n_layers + 1):
            x, (kc, vc), y = ins[l - 1], cs[l - 1], outs[l - 1]
            if self.is_global(l):
                calls.append(("full_decode", lambda x=x, kc=kc, vc=vc, y=y: full_decode(
                    x["q"], x["k"], x["v"], x["wq"], x["wk"], kc, vc, pos, y=y, workspace=workspace,
                    stream=stream, **kw)))
            else:
                if kc.shape[2] != self.window:
                    raise ValueError(f"layer {l}: ring of {kc.shape[2]} slots for window {self.window}")
                calls.append(("gswa_decode", lambda x=x, kc=kc, vc=vc, y=y: gswa_decode(
                    x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], kc, vc, pos, y=y, stream=stream, **kw)))
        return calls

    def decode(self, inputs, caches, pos, outputs, workspace=None, stream=None):
        """Run one decode step through every layer in order (asynchronously)."""
        for _, fn in self.decode_calls(inputs, caches, pos, outputs, workspace, stream):
            fn()
        return outputs
