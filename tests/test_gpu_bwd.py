"""Parity of the CUDA backward (gated sliding window and full causal) with the
float64 oracle's gradients (needs a B200).

The GPU backward consumes the GPU forward's y and lse, as a training step
does; the oracle differentiates its own float64 forward.  Every gradient is
compared element by element (relative L2, tests/parity.py).  Full-size cases
run the whole workload on the GPU and compare one (sequence, KV head) group,
whose q/k/v/g gradients depend on that group's inputs only."""
import pytest
import torch

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_grad_close, assert_weight_grad_close
from workloads import WORKLOADS, Shape, attention_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_512": (WORKLOADS["tiny"], 0, False),
    "ragged_200_gqa2": (Shape(B=2, T=200, Hq=8, Hkv=2), 1, True),
    "single_token": (Shape(B=3, T=1, Hq=4, Hkv=1), 3, False),
    "T33": (Shape(B=1, T=33, Hq=4, Hkv=1), 4, True),
    "T1000_tiles": (Shape(B=1, T=1000, Hq=8, Hkv=2), 5, False),
    "window_1": (Shape(B=1, T=150, Hq=4, Hkv=1, window=1), 6, True),
    "window_64": (Shape(B=1, T=300, Hq=4, Hkv=1, window=64), 7, False),
    "window_100": (Shape(B=2, T=333, Hq=4, Hkv=1, window=100), 8, True),
    "rope_0": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=0), 9, False),
    "rope_64": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=64), 10, True),
    "rope_128": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=128), 11, True),
    "base_1e7": (Shape(B=1, T=700, Hq=8, Hkv=2, rope_base=1e7), 12, False),
}


def gpu_swa(s, x):
    kw = dict(window=s.window, rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    y, lse = gca.gswa_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], **kw)
    out = gca.gswa_bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], y, lse, x["dy"], **kw)
    assert gca.gswa_check_status() == 0
    return out


def gpu_full(s, x):
    kw = dict(rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    y, lse = gca.full_attn_fwd(x["q"], x["k"], x["v"], x["wq"], x["wk"], **kw)
    out = gca.full_attn_bwd(x["q"], x["k"], x["v"], x["wq"], x["wk"], y, lse, x["dy"], **kw)
    assert gca.gswa_check_status() == 0
    return out


def oracle_bwd(s, x, gated):
    return oracle.attn_bwd(x["q"], x["k"], x["v"], x["g"] if gated else None, x["wq"], x["wk"], x["dy"],
                           window=s.window if gated else 0, gated=gated, **oracle.shape_kwargs(s))


@pytest.mark.parametrize("name", sorted(CASES))
def test_gswa_bwd_matches_oracle(name):
    s, seed, rw = CASES[name]
    x = attention_inputs(s, seed, random_weights=rw, with_grad=True)
    dq, dk, dv, dg, dwq, dwk = gpu_swa(s, {n: t.cuda() for n, t in x.items()})
    oq, ok, ov, og, owq, owk = oracle_bwd(s, x, True)
    for got, ref, what in ((dq, oq, "dq"), (dk, ok, "dk"), (dv, ov, "dv"), (dg, og, "dg")):
        assert_grad_close(got, ref, what)
    assert_weight_grad_close(dwq, owq, "dw_q")
    assert_weight_grad_close(dwk, owk, "dw_k")


@pytest.mark.parametrize("name", sorted(n for n in CASES if not n.startswith("window")))
def test_full_bwd_matches_oracle(name):
    s, seed, rw = CASES[name]
    x = attention_inputs(s, seed, random_weights=rw, with_grad=True)
    dq, dk, dv, dwq, dwk = gpu_full(s, {n: t.cuda() for n, t in x.items()})
    oq, ok, ov, _, owq, owk = oracle_bwd(s, x, False)
    for got, ref, what in ((dq, oq, "dq"), (dk, ok, "dk"), (dv, ov, "dv")):
        assert_grad_close(got, ref, what)
    assert_weight_grad_close(dwq, owq, "dw_q")
    assert_weight_grad_close(dwk, owk, "dw_k")


def test_bwd_deterministic():
    """The gated backward is bit-reproducible (no global atomics, fixed-order dw
    sums).  The full causal backward keeps dk, dv and dw_k bit-reproducible; its
    dq~ is an f32 sum whose atomic adds from different key tiles land in any
    order, so dq and dw_q may differ in their last bits between runs."""
    s = Shape(B=2, T=600, Hq=8, Hkv=2)
    x = {n: t.cuda() for n, t in attention_inputs(s, 20, random_weights=True, with_grad=True).items()}
    a, b = gpu_swa(s, x), gpu_swa(s, x)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    (dq1, dk1, dv1, dwq1, dwk1), (dq2, dk2, dv2, dwq2, dwk2) = gpu_full(s, x), gpu_full(s, x)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2) and torch.equal(dwk1, dwk2)
    for u, v in ((dq1, dq2), (dwq1, dwq2)):
        u, v = u.double(), v.double()
        assert ((u - v).norm() / v.norm()).item() <= 1e-3


def _group(t, b, kvh, heads):
    return t[b:b + 1, :, kvh * heads:(kvh + 1) * heads].contiguous()


@pytest.mark.parametrize("workload,gated", [("train_4k", True), ("train_4k", False), ("prefill_64k", True)])
def test_bwd_full_size_one_group(workload, gated):
    s = WORKLOADS[workload]
    x = attention_inputs(s, 0, device="cuda", with_grad=True)
    if gated:
        dq, dk, dv, dg, _, _ = gpu_swa(s, x)
    else:
        dq, dk, dv, _, _ = gpu_full(s, x)
    b, kvh = s.B - 1, s.Hkv // 2
    xs = {n: (_group(t, b, kvh, 4) if n in ("q", "g", "dy") else _group(t, b, kvh, 1) if n in ("k", "v") else t)
          for n, t in x.items()}
    xs = {n: t.cpu() for n, t in xs.items()}
    sg = s.replace(B=1, Hq=4, Hkv=1)
    oq, ok, ov, og, _, _ = oracle_bwd(sg, xs, gated)
    assert_grad_close(_group(dq, b, kvh, 4), oq, "dq")
    assert_grad_close(_group(dk, b, kvh, 1), ok, "dk")
    assert_grad_close(_group(dv, b, kvh, 1), ov, "dv")
    if gated:
        assert_grad_close(_group(dg, b, kvh, 4), og, "dg")


def test_bwd_empty_writes_zero_weight_grads():
    s = Shape(B=1, T=0, Hq=4, Hkv=1)
    x = attention_inputs(s, 0, device="cuda", with_grad=True)
    y = torch.empty_like(x["q"])
    lse = torch.empty((1, 4, 0), dtype=torch.float32, device="cuda")
    _, _, _, _, dwq, dwk = gca.gswa_bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], y, lse, x["dy"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(dwq) == 0 and torch.count_nonzero(dwk) == 0
