"""Parity of whole attention stacks with the float64 oracle, layer by layer
(needs a B200).

ZGCM-1 §2.1 Model overview: 32 layers, global (full causal, ungated) at
1-based layers 6, 12, 18, 24, 30 and gated sliding-window elsewhere; the
Figure 3 caption puts the last global layer at 29 counted from 0.  The stack
driver (global_causal_attention_b200.stack) routes every layer to its entry
point; these tests give each layer its own inputs (and, in decode, its own
cache) so that a layer sent to the wrong entry point, the wrong cache or the
wrong position shows up as a mismatch in that layer."""
import numpy as np
import pytest
import torch

import oracle
from global_causal_attention_b200.stack import AttentionStack, global_layers
from tests.parity import assert_fwd_close
from workloads import GLOBAL_LAYERS_1BASED, N_LAYERS, Shape, attention_inputs, decode_inputs

pytestmark = pytest.mark.gpu


def test_prefill_stack_matches_oracle_every_layer():
    s = Shape(B=1, T=1024, Hq=8, Hkv=2)
    st = AttentionStack(n_layers=N_LAYERS, window=s.window, rope_dims=s.rope_dims, rope_base=s.rope_base,
                        eps=s.eps, scale=s.scale)
    assert tuple(sorted(st.globals)) == GLOBAL_LAYERS_1BASED
    ins_cpu = [attention_inputs(s, 100 + l, random_weights=(l % 3 == 0)) for l in range(1, N_LAYERS + 1)]
    ins = [{n: t.cuda() for n, t in x.items()} for x in ins_cpu]
    outs = [(torch.empty_like(x["q"]), torch.empty(s.B, s.Hq, s.T, dtype=torch.float32, device="cuda"))
            for x in ins]
    st.prefill(ins, outs)
    import global_causal_attention_b200 as gca
    assert gca.gswa_check_status() == 0
    for l in range(1, N_LAYERS + 1):
        x = ins_cpu[l - 1]
        glob = st.is_global(l)
        yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], None if glob else x["g"], x["wq"], x["wk"],
                                 window=0 if glob else s.window, gated=not glob, **oracle.shape_kwargs(s))
        y, lse = outs[l - 1]
        assert_fwd_close(y, yo, f"layer {l} y")
        assert_fwd_close(lse, lo, f"layer {l} lse")


def _bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def test_decode_stack_matches_oracle_every_layer_two_steps():
    """Two consecutive decode steps through the 32-layer stack: B = 4 sequences
    at positions straddling the ring wrap (0, 127, 128, 5000, then each + 1),
    a 128-slot ring per sliding-window layer and an 8,192-token linear cache
    per global layer, distinct inputs and caches in every layer.  The oracle's
    caches are advanced with the oracle's own prepared key (rounded to bf16,
    as the cache stores it) and the raw value, so step 2 checks that every
    layer reads the token its own step-1 call wrote."""
    B, Hq, Hkv, D, W, Tmax = 4, 8, 2, 128, 128, 8192
    st = AttentionStack(n_layers=N_LAYERS, window=W, rope_dims=42, rope_base=1e4, eps=1e-6)
    kw = dict(rope_dims=42, rope_base=1e4, eps=1e-6, scale=D ** -0.5)
    host = []     # per layer: inputs of both steps and the oracle's caches
    for l in range(1, N_LAYERS + 1):
        n = Tmax if st.is_global(l) else W
        x1 = decode_inputs(B, Hq, Hkv, D, n, seed=200 + l, random_weights=(l % 2 == 0))
        x2 = decode_inputs(B, Hq, Hkv, D, 1, seed=300 + l)
        host.append(dict(step=[x1, {**x2, "wq": x1["wq"], "wk": x1["wk"]}],
                         kc=x1["k_cache"].clone(), vc=x1["v_cache"].clone()))
    dev_caches = [(h["kc"].cuda(), h["vc"].cuda()) for h in host]
    positions = [torch.tensor([0, 127, 128, 5000], dtype=torch.int64)]
    positions.append(positions[0] + 1)
    import global_causal_attention_b200 as gca
    for step, pos in enumerate(positions):
        ins = [{n: h["step"][step][n].cuda() for n in ("q", "k", "v", "g", "wq", "wk")} for h in host]
        outs = [torch.empty(B, Hq, D, dtype=torch.bfloat16, device="cuda") for _ in host]
        st.decode(ins, dev_caches, pos.cuda(), outs)
        assert gca.gswa_check_status() == 0
        for l in range(1, N_LAYERS + 1):
            h = host[l - 1]
            x = h["step"][step]
            glob = st.is_global(l)
            yo, kp = oracle.decode(x["q"], x["k"], x["v"], None if glob else x["g"], x["wq"], x["wk"], h["kc"],
                                   h["vc"], pos.numpy(), window=0 if glob else W, gated=not glob, **kw)
            assert_fwd_close(outs[l - 1], yo, f"step {step} layer {l} y")
            # advance the oracle's cache as the library's contract says (c13: prepared key, raw value)
            kpb = _bf16_round(kp)
            for b, p in enumerate(pos.tolist()):
                row = p if glob else p % W
                h["kc"][b, :, row] = kpb[b]
                h["vc"][b, :, row] = x["v"][b]
            # the device cache holds the same values (the key up to one bf16 rounding step)
            kc, vc = dev_caches[l - 1]
            for b, p in enumerate(pos.tolist()):
                row = p if glob else p % W
                assert torch.equal(vc[b, :, row].cpu(), x["v"][b]), f"layer {l} v row"
                assert (kc[b, :, row].cpu().double() - h["kc"][b, :, row].double()).abs().max() <= 2e-2


def test_schedules_of_the_hybrid_experiments():
    """§2.2 compares 1:1, 3:1 and 5:1 sliding-window:global schedules; the
    stack runs each (32 layers, T = 256, one layer of each kind checked)."""
    s = Shape(B=1, T=256, Hq=4, Hkv=1)
    import global_causal_attention_b200 as gca
    for r in (1, 3, 5):
        st = AttentionStack(n_layers=N_LAYERS, swa_per_global=r, window=s.window, rope_dims=s.rope_dims,
                            rope_base=s.rope_base, eps=s.eps, scale=s.scale)
        assert len(st.globals) == N_LAYERS // (r + 1)
        x = attention_inputs(s, 7 + r)
        xd = {n: t.cuda() for n, t in x.items()}
        outs = [(torch.empty_like(xd["q"]), torch.empty(1, 4, s.T, dtype=torch.float32, device="cuda"))
                for _ in range(N_LAYERS)]
        st.prefill(xd, outs)
        assert gca.gswa_check_status() == 0
        first_global = min(global_layers(N_LAYERS, r))
        for l in (1, first_global):
            glob = st.is_global(l)
            yo, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], None if glob else x["g"], x["wq"], x["wk"],
                                    window=0 if glob else s.window, gated=not glob, **oracle.shape_kwargs(s))
            assert_fwd_close(outs[l - 1][0], yo, f"{r}:1 layer {l}")
