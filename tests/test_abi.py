"""The C ABI library: builds, loads without a GPU, exports every declared symbol,
and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

import global_causal_attention_b200 as gca
from global_causal_attention_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gca.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_strerror(L):
    assert gca.strerror(0) == "ok"
    assert "timed out" in gca.strerror(-6)


def test_kv_cache_bytes_matches_pages():
    # ZGCM-1 §2.3: 4 KiB per token per layer, 128 KiB all-global, 32.0 / 5.0 GiB at 256K
    assert gca.gswa_kv_cache_bytes(1, 0, 128, 8, 128, 2, 1) == 4096
    assert gca.gswa_kv_cache_bytes(32, 0, 128, 8, 128, 2, 1) == 128 * 1024
    assert gca.gswa_kv_cache_bytes(32, 0, 128, 8, 128, 2, 262144) == 32 * 2**30
    hyb = gca.gswa_kv_cache_bytes(5, 27, 128, 8, 128, 2, 262144)
    assert abs(hyb / 2**30 - 5.0) < 0.05
    assert gca.gswa_kv_cache_bytes(-1, 0, 128, 8, 128, 2, 1) == -1


def _call_fwd(L, s, ptr=16):
    return L.gswa_fwd(ctypes.byref(s), ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, None, 0, None)


@pytest.mark.parametrize("field,value,code", [
    ("D", 64, -2), ("Hq", 6, -2), ("window", 0, -2), ("window", 129, -2), ("rope_dims", 43, -2),
    ("rope_dims", 130, -2), ("B", -1, -1), ("eps", -1.0, -1),
])
def test_host_validation(L, field, value, code):
    s = gca.make_shape(1, 64, 4, 1)
    setattr(s, field, value)
    assert _call_fwd(L, s) == code


def test_null_and_misaligned_pointers(L):
    s = gca.make_shape(1, 64, 4, 1)
    assert L.gswa_fwd(None, 16, 16, 16, 16, 16, 16, 16, None, None, 0, None) == -1
    assert L.gswa_fwd(ctypes.byref(s), None, 16, 16, 16, 16, 16, 16, None, None, 0, None) == -1
    assert _call_fwd(L, s, ptr=18) == -3


def test_fwd_workspace_holds_the_prepared_keys(L):
    s = gca.make_shape(2, 100, 8, 2)
    # k~ [B, T, Hkv, D] bf16, rounded up to 256 bytes
    assert gca.workspace_bytes(gca.OP_GSWA_FWD, s) == -(-2 * 100 * 2 * 128 * 2 // 256) * 256
    need = gca.workspace_bytes(gca.OP_GSWA_FWD, s)
    assert L.gswa_fwd(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, None, None, 0, None) == -4
    assert L.gswa_fwd(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, None, 16, need - 1, None) == -4
    assert L.gswa_fwd(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, None, 24, need, None) == -3


def test_empty_problem_is_a_no_op(L):
    s = gca.make_shape(0, 64, 4, 1)
    assert _call_fwd(L, s, ptr=0) == 0


def declared_arity():
    """Parameter count of every function declared in include/*.h."""
    out = {}
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(([^)]*)\)\s*;", text, flags=re.M):
                params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
                out[m.group(1)] = len(params)
    return out


def test_binding_signatures_match_header(L):
    """Every ctypes signature of the binding has the header's parameter count
    (a short signature silently truncates the trailing stream handle)."""
    arity = declared_arity()
    for name, args in L._gswa_signatures.items():
        assert arity[name] == len(args), (name, arity[name], len(args))


def _a256(x):
    return -(-x // 256) * 256


@pytest.mark.parametrize("B,T,Hq,Hkv", [(1, 64, 4, 1), (2, 100, 8, 2), (8, 4096, 32, 8)])
def test_workspace_sizes_follow_the_buffer_layouts(B, T, Hq, Hkv):
    """gswa_workspace_bytes against the layouts the header documents (host
    code only): bf16 [B,T,H,128] tensors, f32-pair row records [B,Hkv,Tp,4],
    per-warp dw partials for up to 256 CTAs, each buffer 256-byte aligned."""
    s = gca.make_shape(B, T, Hq, Hkv)
    q, k = B * T * Hq * 128 * 2, B * T * Hkv * 128 * 2
    Tp = -(-T // 32) * 32
    rec = B * Hkv * Tp * 4 * 8
    part = _a256(256 * 4 * 128 * 4)
    assert gca.workspace_bytes(gca.OP_GSWA_FWD, s) == _a256(k)                      # k~
    assert gca.workspace_bytes(gca.OP_FULL_FWD, s) == _a256(k) + _a256(q)           # k~, q~
    assert gca.workspace_bytes(gca.OP_GSWA_BWD, s) == _a256(q) + _a256(k) + _a256(q) + _a256(rec) + 2 * part
    # full causal: q~, k~, records, the f32 dq~ accumulator, dw_q partials of the dq post pass
    # (512 CTAs x 8 warps) and dw_k partials of the fused kernel (256 CTAs x 4 warps)
    assert gca.workspace_bytes(gca.OP_FULL_BWD, s) == (_a256(q) + _a256(k) + _a256(rec) + _a256(2 * q)
                                                        + _a256(512 * 8 * 128 * 4) + _a256(256 * 4 * 128 * 4))
    assert gca.workspace_bytes(gca.OP_GSWA_DECODE, s) == 0


def test_full_decode_workspace_and_the_fixed_scratch():
    # q~ in f32 [B,Hq,128] + partials [B,Hkv,chunks of 4096 keys,4 heads,(4 + 128) f32]
    for B, Hq, Hkv, Tmax in [(1, 4, 1, 1), (4, 8, 2, 10000), (32, 32, 8, 262144)]:
        s = gca.make_shape(B, 1, Hq, Hkv, cache_len=Tmax)
        nch = -(-Tmax // 4096)
        want = _a256(B * Hq * 128 * 4) + _a256(B * Hkv * nch * 4 * 132 * 4)
        assert gca.workspace_bytes(gca.OP_FULL_DECODE, s) == want
    # the 32-sequence, 262,144-token decode fits the 36 MiB allocation-free scratch
    assert want <= 36 << 20
