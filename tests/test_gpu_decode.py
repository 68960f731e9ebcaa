"""Parity of the CUDA decode steps (ring cache and linear cache) with the float64
oracle, and their cache updates (needs a B200)."""
import numpy as np
import pytest
import torch

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_fwd_close
from workloads import DECODE_256K, Shape, decode_inputs, fill_randn_bf16_

pytestmark = pytest.mark.gpu


def _kw(R=42, base=1e4):
    s = Shape(B=1, T=1, Hq=4, Hkv=1, rope_dims=R, rope_base=base)
    return dict(rope_dims=R, rope_base=base, eps=s.eps, scale=s.scale)


@pytest.mark.parametrize("W,positions,R", [(128, [0, 5, 126, 127, 128, 1000, 262143], 42),
                                           (16, [0, 15, 16, 17, 300], 42),
                                           (128, [3, 200], 0),
                                           (100, [0, 99, 100, 101, 5000], 42),
                                           (37, [36, 37, 73], 64),
                                           (1, [0, 7], 42)])
def test_swa_decode_matches_oracle(W, positions, R):
    B, Hq, Hkv = len(positions), 8, 2
    x = decode_inputs(B, Hq, Hkv, 128, W, seed=W + R, random_weights=True)
    pos = torch.tensor(positions, dtype=torch.int64)
    kw = _kw(R, 1e7 if max(positions) > 100000 else 1e4)
    xd = {n: t.cuda() for n, t in x.items()}
    kc, vc = xd["k_cache"].clone(), xd["v_cache"].clone()
    y = gca.gswa_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], kc, vc, pos.cuda(), **kw)
    assert gca.gswa_check_status() == 0
    yo, kp = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], x["k_cache"], x["v_cache"],
                           pos.numpy(), window=W, gated=True, **kw)
    assert_fwd_close(y, yo, "y")
    kc, vc = kc.cpu(), vc.cpu()
    for b, p in enumerate(positions):
        slot = p % W
        assert np.abs(kc[b, :, slot].double().numpy() - kp[b]).max() <= 2e-2
        assert torch.equal(vc[b, :, slot], x["v"][b])
        others = [s for s in range(W) if s != slot]
        assert torch.equal(kc[b, :, others], x["k_cache"][b, :, others])
        assert torch.equal(vc[b, :, others], x["v_cache"][b, :, others])


@pytest.mark.parametrize("Tmax,positions", [(9000, [0, 1, 4095, 4096, 8999]), (4096, [4095, 100]),
                                            (33, [0, 32, 31])])
def test_full_decode_matches_oracle(Tmax, positions):
    B, Hq, Hkv = len(positions), 8, 2
    x = decode_inputs(B, Hq, Hkv, 128, Tmax, seed=Tmax, random_weights=True)
    pos = torch.tensor(positions, dtype=torch.int64)
    kw = _kw()
    xd = {n: t.cuda() for n, t in x.items()}
    kc, vc = xd["k_cache"].clone(), xd["v_cache"].clone()
    y = gca.full_decode(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], kc, vc, pos.cuda(), **kw)
    assert gca.gswa_check_status() == 0
    yo, kp = oracle.decode(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], x["k_cache"], x["v_cache"],
                           pos.numpy(), window=0, gated=False, **kw)
    assert_fwd_close(y, yo, "y")
    for b, p in enumerate(positions):
        assert np.abs(kc[b, :, p].double().cpu().numpy() - kp[b]).max() <= 2e-2
        assert torch.equal(vc[b, :, p].cpu(), x["v"][b])


def test_decode_position_out_of_range_is_reported():
    x = decode_inputs(2, 4, 1, 128, 64, seed=3)
    xd = {n: t.cuda() for n, t in x.items()}
    kc, vc = xd["k_cache"].clone(), xd["v_cache"].clone()
    gca.full_decode(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], kc, vc,
                    torch.tensor([64, 3], dtype=torch.int64, device="cuda"))
    assert gca.gswa_check_status() == -1   # GSWA_ERR_INVALID_ARG: a position outside the cache
    assert torch.equal(kc[0], xd["k_cache"][0])   # sequence 0 (position 64 >= Tmax) skipped
    kc2 = xd["k_cache"].clone()
    gca.gswa_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], kc2, vc,
                    torch.tensor([-1, 3], dtype=torch.int64, device="cuda"))
    assert gca.gswa_check_status() == -1
    assert torch.equal(kc2[0], xd["k_cache"][0])


def test_full_decode_full_size_sampled():
    """Batch 32 at position 262143 over 262144-token caches (one global layer:
    16 GiB each for K and V); the oracle checks sampled (sequence, kv head) pairs."""
    c = DECODE_256K
    B, Hq, Hkv, D, Tmax = c["B"], c["Hq"], c["Hkv"], c["D"], c["Tmax"]
    kc = torch.empty((B, Hkv, Tmax, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    fill_randn_bf16_(kc, 21)
    fill_randn_bf16_(vc, 22)
    x = decode_inputs(B, Hq, Hkv, D, 1, seed=23)
    xd = {n: t.cuda() for n, t in x.items() if n not in ("k_cache", "v_cache")}
    pos = torch.full((B,), c["pos"], dtype=torch.int64, device="cuda")
    kw = _kw(c["rope_dims"], c["rope_base"])
    kc_before = {(b, h): (kc[b, h].cpu(), vc[b, h].cpu()) for b, h in [(0, 0), (31, 7), (17, 3)]}
    y = gca.full_decode(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], kc, vc, pos, **kw)
    assert gca.gswa_check_status() == 0
    for (b, h), (kb, vb) in kc_before.items():
        sl = slice(4 * h, 4 * h + 4)
        yo, _ = oracle.decode(x["q"][b:b + 1, sl], x["k"][b:b + 1, h:h + 1], x["v"][b:b + 1, h:h + 1], None,
                              x["wq"], x["wk"], kb[None, None], vb[None, None], [c["pos"]], window=0,
                              gated=False, **kw)
        assert_fwd_close(y[b:b + 1, sl], yo, f"y[{b},{h}]")
    del kc, vc
    torch.cuda.empty_cache()
