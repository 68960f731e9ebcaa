"""Parity of the CUDA gated-SWA forward with the float64 oracle (needs a B200)."""
import pytest
import torch

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_fwd_close
from workloads import WORKLOADS, Shape, attention_inputs, sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    # name: (shape, seed, random_weights)
    "tiny_512": (WORKLOADS["tiny"], 0, False),
    "ragged_200_gqa2": (Shape(B=2, T=200, Hq=8, Hkv=2), 1, True),
    "ragged_37_w16": (Shape(B=1, T=37, Hq=4, Hkv=1, window=16), 2, True),
    "single_token": (Shape(B=3, T=1, Hq=4, Hkv=1), 3, False),
    "window_1": (Shape(B=2, T=100, Hq=4, Hkv=1, window=1), 4, True),
    "window_64_T161": (Shape(B=1, T=161, Hq=8, Hkv=2, window=64), 5, False),
    "rope_0": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=0), 6, False),
    "rope_64": (Shape(B=2, T=130, Hq=4, Hkv=1, rope_dims=64), 12, True),
    "rope_128": (Shape(B=1, T=300, Hq=4, Hkv=1, rope_dims=128), 7, True),
    "base_1e7_T1000": (Shape(B=1, T=1000, Hq=8, Hkv=2, rope_base=1e7), 8, False),
    "many_strips_T96": (Shape(B=5, T=96, Hq=12, Hkv=3), 9, True),
}


def run_gpu(s, x):
    xd = {n: t.cuda() for n, t in x.items()}
    y, lse = gca.gswa_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], window=s.window,
                          rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    assert gca.gswa_check_status() == 0
    return y, lse


@pytest.mark.parametrize("name", sorted(CASES))
def test_swa_fwd_matches_oracle(name):
    s, seed, rw = CASES[name]
    x = attention_inputs(s, seed, random_weights=rw)
    y, lse = run_gpu(s, x)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                             gated=True, **oracle.shape_kwargs(s))
    assert_fwd_close(y, yo, "y")
    assert_fwd_close(lse, lo, "lse")


@pytest.mark.parametrize("name", ["tiny_512", "window_64_T161", "ragged_37_w16"])
def test_swa_fwd_exact_max_path(name):
    """One-dimension weight spikes (max|w| = 4, other weights 1) put the QK-norm
    score bound past the range where the kernel uses it as the softmax
    reference, so the exact row-max pass runs; the scores stay close to those
    of unit weights."""
    s, seed, _ = CASES[name]
    x = attention_inputs(s, seed)
    wq, wk = torch.ones(128), torch.ones(128)
    wq[9], wk[100] = 4.0, 4.0
    x["wq"], x["wk"] = wq.to(torch.bfloat16), wk.to(torch.bfloat16)
    y, lse = run_gpu(s, x)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window, gated=True,
                             **oracle.shape_kwargs(s))
    assert_fwd_close(y, yo, "y")
    assert_fwd_close(lse, lo, "lse")


def test_swa_fwd_deterministic():
    s = Shape(B=2, T=257, Hq=8, Hkv=2)
    x = attention_inputs(s, 11)
    y1, l1 = run_gpu(s, x)
    y2, l2 = run_gpu(s, x)
    assert torch.equal(y1, y2) and torch.equal(l1, l2)


@pytest.mark.parametrize("workload,nrows", [("train_4k", 48), ("prefill_64k", 24), ("prefill_256k", 16)])
def test_swa_fwd_full_size_sampled_rows(workload, nrows):
    """The full workload in the launch configuration the benchmark times; the oracle
    evaluates a seeded sample of query rows (all heads, all sequences)."""
    s = WORKLOADS[workload]
    x = attention_inputs(s, 0, device="cuda")
    y, lse = gca.gswa_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                          rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    assert gca.gswa_check_status() == 0
    rows = sample_rows(s.T, nrows, seed=1)
    yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                             gated=True, rows=rows.numpy(), **oracle.shape_kwargs(s))
    assert_fwd_close(y[:, rows.cuda()], yo, "y")
    assert_fwd_close(lse[:, :, rows.cuda()], lo, "lse")


def test_gate_precision_window_1():
    """With window 1 each row attends to its own key only (P = 1), so the
    kernel's output is bf16(v ⊙ σ~(g)) and its error against the exact
    v ⊙ σ(g) is the gate's evaluation error plus the final bf16 rounding.
    The kernel evaluates σ in f32 and keeps it as f16 until the product;
    the error that adds, in quadrature on top of the unavoidable rounding of
    the output to bf16, must stay well below that rounding."""
    s = Shape(B=2, T=2048, Hq=8, Hkv=2, window=1)
    x = attention_inputs(s, 21)
    # one-dimension weight spikes select the exact row-max path, where the one
    # visible score is its own maximum, so P = 2^0 = 1 and l = 1 exactly: no
    # rounding of P enters the output, only the gate's and the output's
    wq, wk = torch.ones(128), torch.ones(128)
    wq[9], wk[100] = 4.0, 4.0
    x["wq"], x["wk"] = wq.to(torch.bfloat16), wk.to(torch.bfloat16)
    y, _ = run_gpu(s, x)
    v = x["v"].double().repeat_interleave(4, dim=2)
    exact = v * torch.sigmoid(x["g"].double())
    best = exact.to(torch.bfloat16).double()          # the exact value, rounded once to bf16
    yd = y.double().cpu()
    nrm = exact.norm().item()
    e_gpu = (yd - exact).norm().item() / nrm
    e_round = (best - exact).norm().item() / nrm
    e_gate = max(e_gpu ** 2 - e_round ** 2, 0.0) ** 0.5
    print(f"gate precision: rel-L2 vs exact {e_gpu:.3e}; bf16 rounding alone {e_round:.3e}; "
          f"gate evaluation (in quadrature) {e_gate:.3e}; max |y - exact| {(yd - exact).abs().max().item():.3e}")
    assert e_gpu <= 5e-3
    assert e_gate <= 0.5 * e_round
