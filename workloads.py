"""Seeded synthetic workloads shared by the tests, the oracle checks and bench.py.

This module holds the shapes of the workloads and the random-number recipes
that fill them, and nothing of the attention arithmetic itself: no norm, no
rotation, no softmax, no gate.  Both the CUDA path and the float64 oracle are
fed from here, so the two sides always see bit-identical bf16 inputs.

Workloads (ZGCM-1, §2.1 model overview: 32 query / 8 KV heads, head dim 128,
128-token window, QK-RMSNorm, partial RoPE with rotary fraction 0.33; §3.2
mid-training: RoPE base 10M for the 256K stage):

* ``tiny``        B=1, T=512, 4 q / 1 kv heads, base 1e4 (correctness case)
* ``train_4k``    B=8, T=4096, 32 q / 8 kv heads, base 1e4 (one layer at the
                  training shape of §2.2, forward and backward)
* ``prefill_64k`` B=1, T=65536, base 1e7
* ``prefill_256k`` B=1, T=262144, base 1e7
* ``decode_256k`` B=32, one new token per sequence at position 262143,
                  caches of 262144 tokens, base 1e7

Values are N(0, 1) drawn in float32 and rounded to bf16; the norm weights are
ones.  Nothing here reads a dataset.
"""
from __future__ import annotations

import dataclasses
import math

import torch

HEAD_DIM = 128
WINDOW = 128
# 0.33 of 128 dims rounded to an even count: floor(42.24) = 42.
ROPE_DIMS = 42
EPS = 1e-6
N_LAYERS = 32
GLOBAL_LAYERS_1BASED = (6, 12, 18, 24, 30)


@dataclasses.dataclass(frozen=True)
class Shape:
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int = HEAD_DIM
    window: int = WINDOW
    rope_dims: int = ROPE_DIMS
    rope_base: float = 1e4
    eps: float = EPS

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Shape(B=1, T=512, Hq=4, Hkv=1, rope_base=1e4),
    "train_4k": Shape(B=8, T=4096, Hq=32, Hkv=8, rope_base=1e4),
    "prefill_64k": Shape(B=1, T=65536, Hq=32, Hkv=8, rope_base=1e7),
    "prefill_256k": Shape(B=1, T=262144, Hq=32, Hkv=8, rope_base=1e7),
}

# Decode: batch 32, one query token at position 262143 per sequence.
DECODE_256K = dict(B=32, Hq=32, Hkv=8, D=HEAD_DIM, window=WINDOW, Tmax=262144,
                   pos=262143, rope_dims=ROPE_DIMS, rope_base=1e7, eps=EPS)


def layer_is_global(layer_1based: int) -> bool:
    """True for the five global (full causal) layers of the 32-layer stack."""
    return layer_1based in GLOBAL_LAYERS_1BASED


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) in float32, rounded to bf16.  Deterministic for (shape, seed, device kind)."""
    g = _gen(seed, device)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def attention_inputs(s: Shape, seed: int = 0, device="cpu", random_weights: bool = False,
                     with_grad: bool = False):
    """q, k, v, g, w_q, w_k (and dy when ``with_grad``) for one attention layer.

    Layouts: q, g, dy [B, T, Hq, D]; k, v [B, T, Hkv, D]; w_q, w_k [D]; all bf16.
    Each tensor has its own sub-seed so that changing one shape does not shift
    another tensor's values.
    """
    q = randn_bf16((s.B, s.T, s.Hq, s.D), seed * 16 + 1, device)
    k = randn_bf16((s.B, s.T, s.Hkv, s.D), seed * 16 + 2, device)
    v = randn_bf16((s.B, s.T, s.Hkv, s.D), seed * 16 + 3, device)
    g = randn_bf16((s.B, s.T, s.Hq, s.D), seed * 16 + 4, device)
    if random_weights:
        # Positive weights around 1 so the norm stays well conditioned.
        wq = (1.0 + 0.25 * randn_bf16((s.D,), seed * 16 + 5, device).float()).to(torch.bfloat16)
        wk = (1.0 + 0.25 * randn_bf16((s.D,), seed * 16 + 6, device).float()).to(torch.bfloat16)
    else:
        wq = torch.ones(s.D, dtype=torch.bfloat16, device=device)
        wk = torch.ones(s.D, dtype=torch.bfloat16, device=device)
    out = dict(q=q, k=k, v=v, g=g, wq=wq, wk=wk)
    if with_grad:
        out["dy"] = randn_bf16((s.B, s.T, s.Hq, s.D), seed * 16 + 7, device)
    return out


def decode_inputs(B, Hq, Hkv, D, cache_len, seed: int = 0, device="cpu", random_weights=False):
    """One decode step: new-token q, k, v, g [B, H, D] and a cache of ``cache_len`` slots.

    The cache is [B, Hkv, cache_len, D] bf16 ~ N(0,1); it stands for keys that
    were already normed and rotated when they were written.
    """
    q = randn_bf16((B, Hq, D), seed * 16 + 8, device)
    k = randn_bf16((B, Hkv, D), seed * 16 + 9, device)
    v = randn_bf16((B, Hkv, D), seed * 16 + 10, device)
    g = randn_bf16((B, Hq, D), seed * 16 + 11, device)
    kc = randn_bf16((B, Hkv, cache_len, D), seed * 16 + 12, device)
    vc = randn_bf16((B, Hkv, cache_len, D), seed * 16 + 13, device)
    if random_weights:
        wq = (1.0 + 0.25 * randn_bf16((D,), seed * 16 + 14, device).float()).to(torch.bfloat16)
        wk = (1.0 + 0.25 * randn_bf16((D,), seed * 16 + 15, device).float()).to(torch.bfloat16)
    else:
        wq = torch.ones(D, dtype=torch.bfloat16, device=device)
        wk = torch.ones(D, dtype=torch.bfloat16, device=device)
    return dict(q=q, k=k, v=v, g=g, wq=wq, wk=wk, k_cache=kc, v_cache=vc)


def fill_randn_bf16_(t: torch.Tensor, seed: int, chunk: int = 1 << 27) -> torch.Tensor:
    """Fill a (possibly huge) bf16 tensor in place with N(0,1) values, slice by
    slice, so no float32 copy of the whole tensor is ever held."""
    flat = t.view(-1)
    for i, part in enumerate(flat.split(chunk)):
        g = _gen(seed * 1009 + i, t.device)
        part.copy_(torch.randn(part.numel(), generator=g, device=t.device, dtype=torch.float32))
    return t


def sample_rows(T: int, n: int, seed: int = 0) -> torch.Tensor:
    """A seeded, sorted set of ``n`` distinct query positions in [0, T), always
    including the first and last position and the window edges 127/128."""
    g = _gen(seed + 1000, "cpu")
    fixed = [0, min(T - 1, 127), min(T - 1, 128), T - 1]
    extra = torch.randperm(T, generator=g)[: max(0, n - len(fixed))].tolist()
    return torch.tensor(sorted(set(fixed + extra)), dtype=torch.int64)
