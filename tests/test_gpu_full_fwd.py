"""Parity of the CUDA full causal forward and of the stand-alone QK prologue with
the float64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_fwd_close
from workloads import WORKLOADS, Shape, attention_inputs, randn_bf16, sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_512": (WORKLOADS["tiny"], 0, False),
    "ragged_200_gqa2": (Shape(B=2, T=200, Hq=8, Hkv=2), 1, True),
    "single_token": (Shape(B=3, T=1, Hq=4, Hkv=1), 3, False),
    "T33": (Shape(B=1, T=33, Hq=4, Hkv=1), 4, True),
    "T1024_many_tiles": (Shape(B=2, T=1024, Hq=8, Hkv=2), 5, False),
    "rope_0": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=0), 6, False),
    "rope_64": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=64), 12, True),
    "rope_128": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=128), 7, True),
    "base_1e7_T1000": (Shape(B=1, T=1000, Hq=8, Hkv=2, rope_base=1e7), 8, False),
    "many_strips_T160": (Shape(B=5, T=160, Hq=12, Hkv=3), 9, True),
}


def run_gpu(s, x):
    xd = {n: t.cuda() for n, t in x.items()}
    y, lse = gca.full_attn_fwd(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], rope_dims=s.rope_dims,
                               rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    assert gca.gswa_check_status() == 0
    return y, lse


@pytest.mark.parametrize("name", sorted(CASES))
def test_full_fwd_matches_oracle(name):
    s, seed, rw = CASES[name]
    x = attention_inputs(s, seed, random_weights=rw)
    y, lse = run_gpu(s, x)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False,
                             **oracle.shape_kwargs(s))
    assert_fwd_close(y, yo, "y")
    assert_fwd_close(lse, lo, "lse")


def spiky_weights():
    """Norm weights of 1 except one dimension of 4 in each: the score bound
    D max|w_q| max|w_k| scale log2 e (about 270) is past the range where the kernel
    uses it as a fixed softmax reference, so the running-max path runs, while the
    scores themselves stay close to those of unit weights."""
    wq, wk = torch.ones(128), torch.ones(128)
    wq[5] = 4.0
    wk[77] = 4.0
    return wq.to(torch.bfloat16), wk.to(torch.bfloat16)


@pytest.mark.parametrize("name", ["tiny_512", "ragged_200_gqa2", "T1024_many_tiles", "T33"])
def test_full_fwd_running_max_path(name):
    s, seed, _ = CASES[name]
    x = attention_inputs(s, seed)
    x["wq"], x["wk"] = spiky_weights()
    y, lse = run_gpu(s, x)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False,
                             **oracle.shape_kwargs(s))
    assert_fwd_close(y, yo, "y")
    assert_fwd_close(lse, lo, "lse")


@pytest.mark.parametrize("R,spiky", [(0, False), (42, False), (42, True)])
def test_full_fwd_running_max_rescale(R, spiky):
    """Every query equals a vector u; keys before position 128 equal -u and later
    keys +u.  For rows past 128 the second key tile's scores exceed the first
    tile's max by ~15 (natural units), far past the 2^8 threshold: with spiky
    norm weights (running-max path) the O accumulator is rescaled in TMEM; with
    unit weights the fixed reference covers the whole range."""
    s = Shape(B=1, T=700, Hq=4, Hkv=1, rope_dims=R)
    x = attention_inputs(s, 14)
    if spiky:
        x["wq"], x["wk"] = spiky_weights()
    u = randn_bf16((128,), 15)
    x["q"] = u.expand(s.B, s.T, s.Hq, 128).contiguous()
    k = u.expand(s.B, s.T, s.Hkv, 128).contiguous().clone()
    k[:, :128] = -k[:, :128]
    x["k"] = k
    y, lse = run_gpu(s, x)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False,
                             **oracle.shape_kwargs(s))
    assert_fwd_close(y, yo, "y")
    assert_fwd_close(lse, lo, "lse")


@pytest.mark.parametrize("workload,nrows", [("train_4k", 32), ("prefill_64k", 8), ("prefill_256k", 4)])
def test_full_fwd_full_size_sampled_rows(workload, nrows):
    s = WORKLOADS[workload]
    x = attention_inputs(s, 0, device="cuda")
    y, lse = gca.full_attn_fwd(x["q"], x["k"], x["v"], x["wq"], x["wk"], rope_dims=s.rope_dims,
                               rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    assert gca.gswa_check_status() == 0
    rows = sample_rows(s.T, nrows, seed=2)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False,
                             rows=rows.numpy(), **oracle.shape_kwargs(s))
    assert_fwd_close(y[:, rows.cuda()], yo, "y")
    assert_fwd_close(lse[:, :, rows.cuda()], lo, "lse")


@pytest.mark.parametrize("R,base,pos0", [(42, 1e4, 0), (42, 1e7, 262000), (0, 1e4, 5), (64, 1e4, 17),
                                         (128, 1e4, 3)])
def test_qk_prep_matches_oracle(R, base, pos0):
    x = randn_bf16((3, 77, 8, 128), 40 + R)
    w = (1.0 + 0.25 * randn_bf16((128,), 41).float()).to(torch.bfloat16)
    out = gca.gswa_qk_prep(x.cuda(), w.cuda(), rope_dims=R, rope_base=base, eps=1e-6, pos0=pos0)
    assert gca.gswa_check_status() == 0
    ref = oracle.qk_prep(x, w, R, base, 1e-6, pos0=pos0)
    # a single bf16 rounding of values of magnitude ~1-4
    assert np.abs(out.double().cpu().numpy() - ref).max() <= 2e-2
