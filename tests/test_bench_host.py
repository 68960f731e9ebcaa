"""Host-side arithmetic of bench.py (no GPU): the algorithmic work every
roofline fraction divides by, checked against closed forms written out from
the layouts (bf16 q, k, v, g, y, dy; f32 lse) and against brute-force pair
counts."""
import pytest

import bench
import workloads
from workloads import WORKLOADS, Shape


def brute_pairs(T, W=None):
    """(query, key) pairs with j <= i, and i - j < W for a window W."""
    return sum(1 for i in range(T) for j in range(i + 1) if W is None or i - j < W)


@pytest.mark.parametrize("T,W", [(1, 1), (5, 1), (7, 3), (60, 128), (128, 128), (129, 128), (300, 128)])
def test_pair_counts_match_brute_force(T, W):
    assert bench.swa_pairs(T, W) == brute_pairs(T, W)
    assert bench.causal_pairs(T) == brute_pairs(T)


def test_gswa_fwd_bytes_per_token():
    # q and g read, y written: 3 x 32 heads x 128 x 2 B; k and v read: 2 x 8 x 128 x 2 B;
    # lse written: 32 x 4 B  ->  24,576 + 4,096 + 128 = 28,800 B per token
    s = WORKLOADS["train_4k"]
    assert bench.algorithmic_work("gswa_fwd", s) == ("hbm", 8 * 4096 * 28_800, "GB/s")
    assert 8 * 4096 * 28_800 == 943_718_400


def test_gswa_bwd_bytes_per_token():
    # read q, g, y, dy (4 x 8,192) and k, v (2 x 2,048) and lse (128);
    # write dq, dg (2 x 8,192) and dk, dv (2 x 2,048)  ->  57,472 B per token
    s = WORKLOADS["train_4k"]
    assert bench.algorithmic_work("gswa_bwd", s) == ("hbm", 8 * 4096 * 57_472, "GB/s")


def test_full_attention_flops():
    # forward: QK^T and PV, 2 x 2 x D flops per visible (causal) pair and head
    s = WORKLOADS["train_4k"]
    fwd = 4 * 128 * 8 * 32 * (4096 * 4097 // 2)
    assert fwd == 1_099_780_063_232
    assert bench.algorithmic_work("full_attn_fwd", s) == ("tensor", fwd, "TFLOP/s")
    # backward: dV, dP, dQ, dK (recomputation of S and dP not counted)
    assert bench.algorithmic_work("full_attn_bwd", s) == ("tensor", 2 * fwd, "TFLOP/s")


def test_decode_bytes():
    d = workloads.DECODE_256K
    s = Shape(B=d["B"], T=1, Hq=d["Hq"], Hkv=d["Hkv"], window=d["window"], rope_base=d["rope_base"])
    pos = d["pos"]
    # linear cache: K and V rows 0..pos of 8 heads, plus new q, y (32 heads) and k, v (8 heads)
    per_seq = 2 * 8 * (pos + 1) * 128 * 2 + 2 * 32 * 128 * 2 + 2 * 8 * 128 * 2
    assert bench.algorithmic_work("full_decode", s, pos) == ("hbm", 32 * per_seq, "GB/s")
    assert 32 * per_seq == 34_360_393_728
    # ring: the min(pos + 1, 128) visible slots, plus new q, g, y and k, v
    for p, vis in ((5, 6), (127, 128), (pos, 128)):
        ring = 32 * (2 * 8 * vis * 128 * 2 + 3 * 32 * 128 * 2 + 2 * 8 * 128 * 2)
        assert bench.algorithmic_work("gswa_decode", s, p) == ("hbm", ring, "GB/s")


def test_op_table_fraction():
    """achieved = algorithmic amount / time per call; frac = achieved / peak."""
    s = WORKLOADS["train_4k"]
    step = bench.Step("t", s, s.B * s.T, [("gswa_fwd", None), ("full_attn_fwd", None), ("gswa_fwd", None)], {}, [])
    K = 4
    op_ms = {"gswa_fwd": 2 * K * 0.5, "full_attn_fwd": K * 2.0}   # 0.5 ms and 2.0 ms per call
    pk = dict(hbm_gbs=6536.7, bf16_tflops=1656.9, bf16_tflops_sustained=1387.5)
    t = bench.op_table(step, op_ms, K, pk, (1656.9, "burst"))
    assert t["gswa_fwd"]["calls_per_step"] == 2
    assert t["gswa_fwd"]["achieved"] == pytest.approx(943_718_400 / 0.5e-3 / 1e9)
    assert t["gswa_fwd"]["frac"] == pytest.approx(943_718_400 / 0.5e-3 / 1e9 / 6536.7)
    tf = 1_099_780_063_232 / 2.0e-3 / 1e12
    assert t["full_attn_fwd"]["achieved"] == pytest.approx(tf)
    assert t["full_attn_fwd"]["frac"] == pytest.approx(tf / 1656.9)
    assert t["full_attn_fwd"]["frac_burst"] == pytest.approx(tf / 1656.9)
    assert t["full_attn_fwd"]["frac_sustained"] == pytest.approx(tf / 1387.5)
    assert step.launches() == 2 * bench.LAUNCHES["gswa_fwd"] + bench.LAUNCHES["full_attn_fwd"]


def test_every_entry_point_has_a_launch_count():
    ops = {"gswa_fwd", "gswa_bwd", "full_attn_fwd", "full_attn_bwd", "gswa_decode", "full_decode"}
    assert set(bench.LAUNCHES) == ops
    assert all(n >= 1 for n in bench.LAUNCHES.values())


def test_tensor_peak_follows_the_clocks():
    """Burst peak for a short region or a run at full clocks without the power
    cap; the sustained (power-capped) peak for a long run that hit the cap."""
    pk = dict(bf16_tflops=1656.9, bf16_tflops_sustained=1387.5)
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1320.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(pk, full, 5.0) == (1656.9, "burst")
    assert bench.tensor_peak(pk, capped, 0.2) == (1656.9, "burst")
    assert bench.tensor_peak(pk, capped, 5.0) == (1387.5, "sustained")
    assert bench.tensor_peak(pk, None, 5.0) == (1387.5, "sustained")


def test_stack_schedules():
    """ZGCM-1 §2.1: 32 layers, global at 1-based 6, 12, 18, 24, 30 (Figure 3
    caption: the last global layer is 29 counted from 0); §2.2's 1:1 and 3:1
    schedules put a global layer after every one or three SWA layers."""
    from global_causal_attention_b200.stack import AttentionStack, global_layers
    assert global_layers(32, 5) == workloads.GLOBAL_LAYERS_1BASED == (6, 12, 18, 24, 30)
    assert max(global_layers(32, 5)) - 1 == 29
    assert global_layers(32, 3) == tuple(range(4, 33, 4))
    assert global_layers(32, 1) == tuple(range(2, 33, 2))
    st = AttentionStack()
    kinds = st.kinds()
    assert kinds.count("global") == 5 and kinds.count("swa") == 27
    assert kinds[30:] == ["swa", "swa"]
    assert all(st.is_global(l) == workloads.layer_is_global(l) for l in range(1, 33))


def test_traffic_entries_name_known_workloads_and_calls():
    """Every measured-traffic figure belongs to a workload the bench runs and
    to one of its entry points, and is at least the call's algorithmic bytes
    for the HBM-bound calls (ncu counts every byte moved)."""
    for (name, op), traffic in bench.TRAFFIC.items():
        assert name in bench.WORKLOAD_NAMES
        assert op in bench.LAUNCHES
        assert traffic > 0
        if name == "train_4k":
            bound, work, _ = bench.algorithmic_work(op, WORKLOADS["train_4k"])
            if bound == "hbm":
                assert traffic >= work, (op, traffic, work)


def test_batch_override_reaches_the_reported_config(monkeypatch):
    """--batch replaces the workload's batch, and the JSON line's config shows it."""
    import dataclasses
    monkeypatch.setitem(WORKLOADS, "train_4k", dataclasses.replace(WORKLOADS["train_4k"], B=4))
    cfg = bench.workload_config("train_4k", 1)
    assert cfg["global_batch"] == 4
    assert "B4 T4096" in cfg["workload"]
