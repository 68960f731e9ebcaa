"""full_decode_noalloc: the allocation-free variant of full_decode (needs a B200).

Calls the entry point through the C ABI and compares it with full_decode on
the same inputs, and with the float64 oracle, twice in a row with different
positions (so the second call reuses the fixed scratch the first one wrote),
and checks that the device's free memory does not move across a call.  Kept
in its own file, collected last, so it also runs after every other GPU test
has used the device."""
import ctypes

import numpy as np
import pytest
import torch

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_fwd_close
from workloads import decode_inputs

pytestmark = pytest.mark.gpu

B, HQ, HKV, TMAX = 4, 8, 2, 10000   # three 4096-key chunks


def _inputs():
    x = {n: t.cuda() for n, t in decode_inputs(B, HQ, HKV, 128, TMAX, seed=31, random_weights=True).items()}
    return x


def _call_abi(x, kc, vc, pos, y):
    s = gca.make_shape(B, 1, HQ, HKV, 128, 128, 42, 1e4, 1e-6, cache_len=TMAX)
    p = lambda t: t.data_ptr()
    rc = gca.lib().full_decode_noalloc(ctypes.byref(s), p(x["q"]), p(x["k"]), p(x["v"]), p(x["wq"]), p(x["wk"]),
                                       p(kc), p(vc), p(pos), p(y), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, gca.strerror(rc)
    assert gca.gswa_check_status() == 0


def test_noalloc_matches_full_decode_twice():
    x = _inputs()
    positions = [torch.tensor([TMAX - 1, 0, 4096, 5000], dtype=torch.int64, device="cuda"),
                 torch.tensor([123, TMAX - 1, 8191, 4095], dtype=torch.int64, device="cuda")]
    kc_ref, vc_ref = x["k_cache"].clone(), x["v_cache"].clone()
    kc, vc = x["k_cache"].clone(), x["v_cache"].clone()
    ys = [torch.empty_like(x["q"]) for _ in positions]
    refs = [gca.full_decode(x["q"], x["k"], x["v"], x["wq"], x["wk"], kc_ref, vc_ref, pos) for pos in positions]
    torch.cuda.synchronize()
    # the oracle's view of the cache, advanced by each call as the library's contract says
    # (the prepared key, rounded to bf16 as the cache stores it, and the raw value)
    hk, hv = x["k_cache"].cpu(), x["v_cache"].cpu()
    xc = {n: x[n].cpu() for n in ("q", "k", "v", "wq", "wk")}
    kw = dict(rope_dims=42, rope_base=1e4, eps=1e-6, scale=128 ** -0.5)
    for i, (pos, y, ref) in enumerate(zip(positions, ys, refs)):
        free_before = torch.cuda.mem_get_info()[0]
        _call_abi(x, kc, vc, pos, y)
        torch.cuda.synchronize()
        if i > 0:   # the first call on the device may do its one-time set-up
            assert torch.cuda.mem_get_info()[0] == free_before
        assert_fwd_close(y, ref, f"call {i} vs full_decode")
        yo, kp = oracle.decode(xc["q"], xc["k"], xc["v"], None, xc["wq"], xc["wk"], hk, hv, pos.cpu().numpy(),
                               window=0, gated=False, **kw)
        assert_fwd_close(y, yo, f"call {i} vs oracle")
        kpb = torch.from_numpy(np.ascontiguousarray(kp)).to(torch.bfloat16)
        for b, p in enumerate(pos.tolist()):
            hk[b, :, p] = kpb[b]
            hv[b, :, p] = xc["v"][b]
    assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    x = _inputs()
    # 64 sequences x 8 KV heads x 64 chunks of partials: about 67 MiB > 36 MiB
    s = gca.make_shape(64, 1, 32, 8, 128, 128, 42, 1e4, 1e-6, cache_len=262144)
    assert gca.workspace_bytes(gca.OP_FULL_DECODE, s) > 36 << 20
    p = x["q"].data_ptr()
    rc = gca.lib().full_decode_noalloc(ctypes.byref(s), p, p, p, p, p, p, p, x["q"].data_ptr(), p,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == -9 and gca.ERRORS[rc] == "SCRATCH_LIMIT"
