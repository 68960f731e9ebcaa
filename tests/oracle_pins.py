"""Pins of the float64 oracle against facts that do not come from the oracle.

Each check takes an oracle library handle ``L`` so that the same suite can be
run against copies of the oracle with a mistake planted in them
(tests/test_oracle_plants.py): a plausible slip anywhere in the oracle -- a
dropped term, a flipped sign, an off-by-one window, a wrong head map -- must
make at least one of these checks fail.

What pins what:
  * library reduction: ``dense_reference`` (F.rms_norm, complex RoPE,
    scaled_dot_product_attention with a band mask and GQA, autograd) for the
    forward, the LSE and every gradient;
  * finite differences of the oracle's own forward for the gradients;
  * special cases the pages' definition fixes: window >= T is full causal
    attention times the gate, window 1 returns v_i ⊙ σ(g_i), g = 0 halves the
    output, each query-head group reads only its own KV head, the cache
    footprint printed in §2.3;
  * invariants: unit RMS after the norm, rotation preserves norms and makes
    scores depend only on i - j, constant values pass through softmax,
    outputs lie in the convex hull of the visible values, decode equals the
    prefill row at the same position.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
from tests import dense_reference as dense
from workloads import Shape, attention_inputs, randn_bf16

HERE = os.path.dirname(os.path.abspath(__file__))
f64 = torch.float64

# A small problem that still has several window edges, GQA groups of 4 and a
# rotated slice of 42 dims.
SMALL = Shape(B=2, T=40, Hq=8, Hkv=2, rope_base=1e4)


def _kw(s: Shape, **over):
    d = dict(rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    d.update(over)
    return d


def _inputs(s: Shape, seed=0, random_weights=True):
    return attention_inputs(s, seed, random_weights=random_weights, with_grad=True)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(1e-300, np.abs(b).max()))


def check_library_forward(L):
    """Oracle forward and LSE == dense library formulation (1e-11 relative)."""
    for window, gated, base, R in [(1, True, 1e4, 42), (3, True, 1e4, 42), (16, True, 1e7, 42),
                                   (40, True, 1e4, 42), (0, False, 1e4, 42), (7, False, 1e4, 0),
                                   (5, True, 1e4, 128)]:
        s = SMALL.replace(rope_base=base, rope_dims=R)
        x = _inputs(s, seed=window + 3)
        y, lse = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=window,
                                 gated=gated, L=L, **_kw(s))
        yd, lsed = dense.forward(*[x[n].to(f64) for n in ("q", "k", "v", "g", "wq", "wk")],
                                 window=window, gated=gated, **_kw(s))
        assert _rel(y, yd) < 1e-11, ("y", window, gated, _rel(y, yd))
        assert _rel(lse, lsed) < 1e-11, ("lse", window, gated, _rel(lse, lsed))


def check_library_backward(L):
    """Oracle gradients == autograd of the dense formulation (1e-10 relative)."""
    for window, gated in [(5, True), (0, False), (40, True)]:
        s = SMALL.replace(T=24)
        x = _inputs(s, seed=11 + window)
        got = oracle.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], x["dy"],
                              window=window, gated=gated, L=L, **_kw(s))
        want = dense.gradients(*[x[n].to(f64) for n in ("q", "k", "v", "g", "wq", "wk")],
                               x["dy"].to(f64), window=window, gated=gated, **_kw(s))
        names = ["dq", "dk", "dv", "dg", "dwq", "dwk"]
        for n, a, b in zip(names, got, want):
            if n == "dg" and not gated:
                assert a is None
                continue
            assert _rel(a, b) < 1e-10, (n, window, gated, _rel(a, b))


def check_finite_differences(L):
    """Central differences of sum(y ⊙ dy) on the float64 path vs oracle gradients."""
    s = Shape(B=1, T=10, Hq=4, Hkv=2, window=3, rope_base=1e4)
    x = _inputs(s, seed=5)
    xf = {n: x[n].to(f64).numpy().copy() for n in x}
    kw = _kw(s)
    grads = oracle.attn_bwd(*[xf[n] for n in ("q", "k", "v", "g", "wq", "wk", "dy")],
                            window=s.window, gated=True, L=L, **kw)
    gmap = dict(zip(["q", "k", "v", "g", "wq", "wk"], [grads[0], grads[1], grads[2], grads[3],
                                                       grads[4], grads[5]]))
    rng = np.random.default_rng(0)
    h = 1e-5

    def loss(arrs):
        y, _ = oracle.attn_fwd(*[arrs[n] for n in ("q", "k", "v", "g", "wq", "wk")],
                               window=s.window, gated=True, L=L, **kw)
        return float((y * arrs["dy"]).sum())

    for name in ("q", "k", "v", "g", "wq", "wk"):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in xf[name].shape)
            a = {n: xf[n] for n in xf}
            p = xf[name].copy(); p[idx] += h
            m = xf[name].copy(); m[idx] -= h
            a[name] = p
            lp = loss(a)
            a[name] = m
            lm = loss(a)
            fd = (lp - lm) / (2 * h)
            an = gmap[name][idx]
            scale = max(1.0, float(np.abs(gmap[name]).max()))
            assert abs(fd - an) < 1e-6 * scale, (name, idx, fd, an)


def check_window_ge_T_is_full(L):
    """Window >= T: gated SWA equals full causal attention times σ(g)."""
    s = SMALL
    x = _inputs(s, seed=21)
    args = [x[n] for n in ("q", "k", "v", "g", "wq", "wk")]
    ys, ls = oracle.attn_fwd(*args, window=s.T, gated=True, L=L, **_kw(s))
    yf, lf = oracle.attn_fwd(*args, window=0, gated=False, L=L, **_kw(s))
    sg = 1.0 / (1.0 + np.exp(-x["g"].to(f64).numpy()))
    assert np.abs(ys - yf * sg).max() < 1e-14
    assert np.array_equal(ls, lf)


def check_window_one(L):
    """Window 1: each query sees only itself, so y_i = v_i ⊙ σ(g_i)."""
    s = SMALL
    x = _inputs(s, seed=22)
    y, lse = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=1,
                             gated=True, L=L, **_kw(s))
    G = s.Hq // s.Hkv
    v = x["v"].to(f64).numpy().repeat(G, axis=2)
    sg = 1.0 / (1.0 + np.exp(-x["g"].to(f64).numpy()))
    assert np.abs(y - v * sg).max() < 1e-14


def check_gqa_isolation(L):
    """Changing KV head c changes exactly the query heads c*G .. c*G+G-1."""
    s = SMALL
    x = _inputs(s, seed=23)
    args = [x[n] for n in ("q", "k", "v", "g", "wq", "wk")]
    y0, _ = oracle.attn_fwd(*args, window=6, gated=True, L=L, **_kw(s))
    G = s.Hq // s.Hkv
    for c in range(s.Hkv):
        k2 = x["k"].clone()
        v2 = x["v"].clone()
        k2[:, :, c] = randn_bf16(k2[:, :, c].shape, 99 + c)
        v2[:, :, c] = randn_bf16(v2[:, :, c].shape, 199 + c)
        y1, _ = oracle.attn_fwd(x["q"], k2, v2, x["g"], x["wq"], x["wk"], window=6, gated=True,
                                L=L, **_kw(s))
        changed = [h for h in range(s.Hq) if not np.array_equal(y0[:, :, h], y1[:, :, h])]
        assert changed == list(range(c * G, c * G + G)), (c, changed)


def check_kv_footprint(L):
    """The §2.3 numbers: 4 KiB/token/layer, 128 vs 20 KiB, 32.0/7.0/5.0 GiB, 6.4x."""
    with open(os.path.join(HERE, "golden", "kv_footprint.json")) as f:
        gold = json.load(f)
    Hkv, D, W, bpe, T = gold["Hkv"], gold["D"], gold["window"], gold["bytes_per_elem"], gold["context"]
    one = oracle.kv_bytes(1, 0, W, Hkv, D, bpe, 1, L=L)
    assert one == 4096
    assert oracle.kv_bytes(32, 0, W, Hkv, D, bpe, 1, L=L) == gold["per_token_kib"]["all_global_32"] * 1024
    # per-token growth of the hybrid stack: only the 5 global layers grow with T
    grow = oracle.kv_bytes(5, 27, W, Hkv, D, bpe, T + 1, L=L) - oracle.kv_bytes(5, 27, W, Hkv, D, bpe, T, L=L)
    assert grow == gold["per_token_kib"]["hybrid_5_global"] * 1024
    gib = 2.0 ** 30
    full = oracle.kv_bytes(32, 0, W, Hkv, D, bpe, T, L=L) / gib
    gdn = oracle.kv_bytes(7, 0, W, Hkv, D, bpe, T, L=L) / gib
    hyb = oracle.kv_bytes(5, 27, W, Hkv, D, bpe, T, L=L) / gib
    tol = gold["printed_precision_gib"]
    assert full == gold["at_256k_gib"]["all_global_32"]
    assert gdn == gold["at_256k_gib"]["gdn_3to1_7_global"]
    assert abs(hyb - gold["at_256k_gib"]["hybrid_5_global"]) < tol
    assert round(full / hyb, 1) == gold["reduction_vs_all_global"]
    toy = gold["toy"]
    per_entry = oracle.kv_bytes(1, 0, toy["window"], 1, 1, 1, 1, L=L)  # K+V of one token
    assert oracle.kv_bytes(toy["global_layers"], toy["swa_layers"], toy["window"], 1, 1, 1,
                           toy["tokens"], L=L) == toy["entries"] * per_entry
    assert oracle.kv_bytes(toy["global_layers"] + toy["swa_layers"], 0, toy["window"], 1, 1, 1,
                           toy["tokens"], L=L) == toy["all_global_entries"] * per_entry


def check_rms_unit(L):
    """With w = 1 the normed rows have mean square ms/(ms + eps); rotation keeps it."""
    x = randn_bf16((2, 9, 3, 128), 31)
    w = torch.ones(128, dtype=torch.bfloat16)
    ms = (x.to(f64) ** 2).mean(-1).numpy()
    want = ms / (ms + 1e-6)
    for R in (0, 42):
        out = oracle.qk_prep(x, w, R, 1e4, 1e-6, pos0=7, L=L)
        got = (out ** 2).mean(-1)
        assert np.abs(got - want).max() < 1e-14, R


def check_rope_closed_form(L):
    """Prepared rows == complex-exponential RoPE of F.rms_norm at large positions."""
    x = randn_bf16((1, 6, 2, 128), 32)
    w = (1.0 + 0.25 * randn_bf16((128,), 33).float()).to(torch.bfloat16)
    for pos0, base in [(0, 1e4), (262138, 1e7), (4090, 1e4)]:
        out = oracle.qk_prep(x, w, 42, base, 1e-6, pos0=pos0, L=L)
        pos = torch.arange(pos0, pos0 + 6, dtype=f64)
        want = dense.prep(x.to(f64), w.to(f64), 42, base, 1e-6, pos).numpy()
        assert np.abs(out - want).max() < 1e-10, (pos0, np.abs(out - want).max())
        # dims past the rotated slice are the plain normed values
        plain = oracle.qk_prep(x, w, 0, base, 1e-6, pos0=pos0, L=L)
        assert np.array_equal(out[..., 42:], plain[..., 42:])


def check_rope_relative(L):
    """Scores depend on positions only through i - j (shift by 1000 positions)."""
    x = randn_bf16((1, 12, 1, 128), 34)
    w = torch.ones(128, dtype=torch.bfloat16)
    a = oracle.qk_prep(x, w, 42, 1e4, 1e-6, pos0=5, L=L)[0, :, 0]
    b = oracle.qk_prep(x, w, 42, 1e4, 1e-6, pos0=1005, L=L)[0, :, 0]
    sa = a @ a[::-1].T
    sb = b @ b[::-1].T
    assert np.abs(sa - sb).max() < 1e-10
    assert not np.allclose(a, b)   # the rotation did act


def check_gate_values(L):
    """g = 0 gives exactly half of the ungated output; g = 30 gives it to 1e-12."""
    s = SMALL
    x = _inputs(s, seed=24)
    args = [x[n] for n in ("q", "k", "v")]
    ya, _ = oracle.attn_fwd(*args, x["g"], x["wq"], x["wk"], window=9, gated=False, L=L, **_kw(s))
    z = torch.zeros_like(x["g"])
    y0, _ = oracle.attn_fwd(*args, z, x["wq"], x["wk"], window=9, gated=True, L=L, **_kw(s))
    assert np.array_equal(y0, 0.5 * ya)
    big = torch.full_like(x["g"], 30.0)
    y1, _ = oracle.attn_fwd(*args, big, x["wq"], x["wk"], window=9, gated=True, L=L, **_kw(s))
    assert np.abs(y1 - ya).max() < 1e-12


def check_softmax_properties(L):
    """Constant values pass through unchanged; outputs lie in the visible values' hull."""
    s = SMALL
    x = _inputs(s, seed=25)
    ones = torch.ones_like(x["v"])
    y, _ = oracle.attn_fwd(x["q"], x["k"], ones, x["g"], x["wq"], x["wk"], window=0, gated=False,
                           L=L, **_kw(s))
    assert np.abs(y - 1.0).max() < 1e-13
    W = 5
    y, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=W,
                           gated=False, L=L, **_kw(s))
    v = x["v"].to(f64).numpy()
    G = s.Hq // s.Hkv
    for i in range(s.T):
        lo = max(0, i - W + 1)
        vis = v[:, lo:i + 1]                      # [B, n, Hkv, D]
        vmin = vis.min(axis=1).repeat(G, axis=1)  # [B, Hq, D]
        vmax = vis.max(axis=1).repeat(G, axis=1)
        assert (y[:, i] >= vmin - 1e-12).all() and (y[:, i] <= vmax + 1e-12).all(), i


def check_decode_matches_prefill(L):
    """Decode at position p over a cache filled from the prefill equals prefill row p."""
    W = 16
    s = Shape(B=2, T=70, Hq=4, Hkv=2, window=W, rope_base=1e4)
    x = _inputs(s, seed=26)
    kw = _kw(s)
    yf, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=W,
                            gated=True, L=L, **kw)
    yc, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=0,
                            gated=False, L=L, **kw)
    kp = oracle.qk_prep(x["k"], x["wk"], s.rope_dims, s.rope_base, s.eps, L=L)  # [B,T,Hkv,D]
    v = x["v"].to(f64).numpy()
    rng = np.random.default_rng(3)
    for p in (0, 1, W - 2, W - 1, W, 2 * W - 1, 2 * W, s.T - 1):
        # ring: stale garbage everywhere, then the live window except the new token
        ring_k = rng.standard_normal((s.B, s.Hkv, W, s.D)) * 50
        ring_v = rng.standard_normal((s.B, s.Hkv, W, s.D)) * 50
        for t in range(max(0, p - W + 1), p):
            ring_k[:, :, t % W] = kp[:, t]
            ring_v[:, :, t % W] = v[:, t]
        q_new = x["q"][:, p].to(f64).numpy()
        k_new = x["k"][:, p].to(f64).numpy()
        v_new = v[:, p]
        g_new = x["g"][:, p].to(f64).numpy()
        pos = np.full(s.B, p)
        y, knew = oracle.decode(q_new, k_new, v_new, g_new, x["wq"].to(f64).numpy(),
                                x["wk"].to(f64).numpy(), ring_k, ring_v, pos, window=W,
                                gated=True, L=L, **kw)
        assert np.abs(y - yf[:, p]).max() < 1e-12, ("ring", p)
        assert np.abs(knew - kp[:, p]).max() < 1e-14
        # linear cache: everything before p, garbage after
        lin_k = rng.standard_normal((s.B, s.Hkv, s.T, s.D)) * 50
        lin_v = rng.standard_normal((s.B, s.Hkv, s.T, s.D)) * 50
        lin_k[:, :, :p] = kp[:, :p].transpose(0, 2, 1, 3)
        lin_v[:, :, :p] = v[:, :p].transpose(0, 2, 1, 3)
        y, _ = oracle.decode(q_new, k_new, v_new, g_new, x["wq"].to(f64).numpy(),
                             x["wk"].to(f64).numpy(), lin_k, lin_v, pos, window=0, gated=False,
                             L=L, **kw)
        assert np.abs(y - yc[:, p]).max() < 1e-12, ("linear", p)


def check_dq_vanishes_for_equal_keys(L):
    """Softmax rows of dS sum to zero, so identical keys give dq = 0."""
    s = Shape(B=1, T=12, Hq=2, Hkv=1, rope_dims=0, rope_base=1e4)
    x = _inputs(s, seed=27)
    k = x["k"][:, :1].expand(-1, s.T, -1, -1).contiguous()
    dq = oracle.attn_bwd(x["q"], k, x["v"], x["g"], x["wq"], x["wk"], x["dy"], window=4,
                         gated=True, L=L, **_kw(s))[0]
    assert np.abs(dq).max() < 1e-13


ALL_CHECKS = [check_library_forward, check_library_backward, check_finite_differences,
              check_window_ge_T_is_full, check_window_one, check_gqa_isolation,
              check_kv_footprint, check_rms_unit, check_rope_closed_form, check_rope_relative,
              check_gate_values, check_softmax_properties, check_decode_matches_prefill,
              check_dq_vanishes_for_equal_keys]
