"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

Every plant is a one-line textual edit of oracle/oracle.c compiled into a
temporary library; the committed oracle is never modified.  A plant that no
pin catches would mean that part of the oracle is unpinned.
"""
import os
import shutil
import tempfile

import pytest

import oracle
from oracle import build as obuild
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(obuild.__file__), "oracle.c")

PLANTS = {
    "window_off_by_one": ("int64_t lo = i - window + 1;", "int64_t lo = i - window;"),
    "rope_sign": ("out[p] = a * c - b * s;", "out[p] = a * c + b * s;"),
    "rope_frequency": ("-2.0 * (double)p / (double)R", "-1.0 * (double)p / (double)R"),
    "gqa_interleaved_map": ("int h = kh * G + hh; /* query head h reads kv head h / G */",
                            "int h = hh * Hkv + kh;"),
    "eps_dropped": ("double r = 1.0 / sqrt(ss / (double)D + eps);",
                    "double r = 1.0 / sqrt(ss / (double)D);"),
    "norm_weight_dropped": ("out[d] = w[d] * n;", "out[d] = n;"),
    "gate_sign": ("yo[d] = gated ? acc[d] * sigmoid(ld(g, qrow * D + d)) : acc[d];",
                  "yo[d] = gated ? acc[d] * sigmoid(-ld(g, qrow * D + d)) : acc[d];"),
    "scale_dropped": ("s[j - lo] = scale * dot;", "s[j - lo] = dot;"),
    "lse_without_max": ("lse[((int64_t)b * Hq + h) * nrows + ri] = mx + log(l);",
                        "lse[((int64_t)b * Hq + h) * nrows + ri] = log(l);"),
    "bwd_softmax_D_dropped": ("double ds = p * (dp[j - lo] - Drow);", "double ds = p * dp[j - lo];"),
    "bwd_rope_transpose_sign": ("du[p] = a * c + b * s;", "du[p] = a * c - b * s;"),
    "bwd_gate_derivative": ("dg[row * D + d] = dyd * acc[d] * sg * (1.0 - sg);",
                            "dg[row * D + d] = dyd * acc[d] * sg;"),
    "bwd_norm_projection_dropped": ("dx[d] = r * (w[d] * du[d] - n[d] * m);",
                                    "dx[d] = r * (w[d] * du[d]);"),
    "bwd_dw_uses_raw_input": ("dw_acc[d] += du[d] * n[d];", "dw_acc[d] += du[d];"),
    "bwd_dk_transposed_operand": ("dkt[j * D + d] += scale * ds * qt[d];",
                                  "dkt[j * D + d] += scale * ds * kt[j * D + d];"),
    "decode_ring_slot": ("int64_t slot = window > 0 ? t % window : t;\n                    for (int d = 0; d < D; ++d) dot",
                         "int64_t slot = window > 0 ? (t + 1) % window : t;\n                    for (int d = 0; d < D; ++d) dot"),
    "kv_bytes_k_only": ("int64_t per_token = 2LL * Hkv * D * bytes_per_elem;",
                        "int64_t per_token = 1LL * Hkv * D * bytes_per_elem;"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_plants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_plant_is_caught(name, workdir):
    old, new = PLANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"plant site for {name} not found in oracle.c"
    planted = src.replace(old, new)
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(planted)
    lib_path = obuild.build(path, os.path.join(workdir, f"lib{name}.so"), extra=("-w",))
    L = oracle.lib(lib_path)
    failures = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(L)
        except AssertionError:
            failures.append(check.__name__)
    assert failures, f"no pin caught the planted mistake {name}"
