"""Failure detection on the GPU: a bounded wait that runs out (needs a B200).

Every wait inside the kernels is bounded.  gswa_set_wait_limit_ns() lowers
the bound to 1 ns, so the first wait that has to spin gives up (the MMA
issuer's poll loop always spins while the first tiles load).  The kernel then
raises its abort flag, every role leaves its loop, in-flight copies land,
tensor memory is freed, and gswa_check_status() reports GSWA_ERR_TIMEOUT.
The next call with the normal bound must then be clean and match the
oracle: that shows the status word was cleared and no tensor memory or
barrier state leaked from the aborted launch.  No GPU fault, trap or hang is
involved: the kernels return on their own."""
import pytest

import global_causal_attention_b200 as gca
import oracle
from tests.parity import assert_fwd_close, assert_grad_close
from workloads import WORKLOADS, Shape, attention_inputs

pytestmark = pytest.mark.gpu

TIMEOUT = -6


def _kw(s):
    return dict(rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)


def _run(op, s, xd):
    if op == "gswa_fwd":
        return gca.gswa_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], window=s.window, **_kw(s))
    if op == "full_attn_fwd":
        return gca.full_attn_fwd(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], **_kw(s))
    if op == "gswa_bwd":
        y, lse = gca.gswa_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], window=s.window, **_kw(s))
        return gca.gswa_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["wq"], xd["wk"], y, lse, xd["dy"],
                            window=s.window, **_kw(s))
    y, lse = gca.full_attn_fwd(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], **_kw(s))
    return gca.full_attn_bwd(xd["q"], xd["k"], xd["v"], xd["wq"], xd["wk"], y, lse, xd["dy"], **_kw(s))


@pytest.mark.parametrize("op", ["gswa_fwd", "full_attn_fwd", "gswa_bwd", "full_attn_bwd"])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_clean(op):
    # the aborted call: a shape with many units per CTA, so that some waits
    # (a producer whose ring is full, an epilogue waiting for a whole unit)
    # last well past the 1 ns limit and the device timer's resolution
    big = Shape(B=2, T=4096, Hq=8, Hkv=2)
    xb = attention_inputs(big, 41, device="cuda", with_grad=True)
    assert gca.gswa_check_status() == 0
    gca.gswa_set_wait_limit_ns(1)
    try:
        _run(op, big, xb)
        rc = gca.gswa_check_status()
    finally:
        gca.gswa_set_wait_limit_ns(0)
    assert rc == TIMEOUT, f"{op}: status {rc} after a 1 ns wait limit"
    s = WORKLOADS["tiny"]
    x = attention_inputs(s, 40, with_grad=True)
    xd = {n: t.cuda() for n, t in x.items()}
    # the default bound again: clean status, correct results
    out = _run(op, s, xd)
    assert gca.gswa_check_status() == 0
    gated = op.startswith("gswa")
    w = s.window if gated else 0
    if op.endswith("fwd"):
        yo, lo = oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"] if gated else None, x["wq"], x["wk"], window=w,
                                 gated=gated, **oracle.shape_kwargs(s))
        assert_fwd_close(out[0], yo, f"{op} y")
        assert_fwd_close(out[1], lo, f"{op} lse")
    else:
        ref = oracle.attn_bwd(x["q"], x["k"], x["v"], x["g"] if gated else None, x["wq"], x["wk"], x["dy"],
                              window=w, gated=gated, **oracle.shape_kwargs(s))
        assert_grad_close(out[0], ref[0], f"{op} dq")
        assert_grad_close(out[1], ref[1], f"{op} dk")
        assert_grad_close(out[2], ref[2], f"{op} dv")
