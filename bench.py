"""Benchmark of the ZGCM-1 attention core on B200 (gated SWA + full causal).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload train_4k]
    python bench.py --impl reference ...      (the float64 CPU oracle)

One step = one pass of every kernel of the hot path that the chosen workload
runs, over one batch of seeded synthetic bf16 input (see STEP_OPS).  Prints one
JSON line (rank 0).  With torchrun (N > 1) every rank runs an independent copy
of the workload on its own GPU (the batch is data parallel; the path has no
exchange step), so scaling is weak and `value` counts the tokens of all ranks.

Timing: W untimed steps, then K steps between a barrier + cuda synchronize on
both sides, CUDA events on the launching stream, max over ranks.  The inputs
(> 600 MB for train_4k) are larger than the 126 MB L2, so every step streams
them from HBM.  SM clocks and throttle reasons are sampled (NVML, read-only)
during the timed region.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch

import workloads
from workloads import WORKLOADS

METRIC = "gated-SWA/full attn tokens/s (prefill+bwd, decode) and % of roofline, 1 B200"
UNIT = "tokens/s"

# What one step of each workload runs (one bench line per workload).
#   train_4k      one attention layer at training shape, both kinds on the same
#                 tensors: gated-SWA forward + backward, full causal forward + backward
#   prefill_64k / prefill_256k   the 32-layer attention stack, forward:
#                 27 gated-SWA layers + 5 full causal layers (1-based 6, 12, 18, 24, 30)
#   decode_256k   one decode step of 32 sequences through the 32-layer stack
#                 (27 ring-cache SWA layers, 5 linear-cache global layers)
WORKLOAD_NAMES = ["train_4k", "prefill_64k", "prefill_256k", "decode_256k"]
LAYERS = workloads.N_LAYERS

# Kernel launches of one call of each entry point.
LAUNCHES = {"gswa_fwd": 2, "gswa_bwd": 7, "full_attn_fwd": 3, "full_attn_bwd": 7, "gswa_decode": 1,
            "full_decode": 3}

# DRAM bytes (read + write) of one call, from an ncu capture of the same
# launches (dram__bytes_read.sum + dram__bytes_write.sum summed over the
# call's kernels).  Absent entries are reported as null: not captured for the
# current kernels.
TRAFFIC = {
    ("decode_256k", "full_decode"): 34_430_000_000,  # 34.40 GB read + 0.03 GB written, 3 launches
    # one call's launches at B4 (one ncu pass), x2 for B8: each sequence's work is independent
    ("train_4k", "gswa_fwd"): 959_200_000,
    ("train_4k", "gswa_bwd"): 3_806_400_000,
    ("train_4k", "full_attn_fwd"): 1_403_200_000,
    ("train_4k", "full_attn_bwd"): 12_171_400_000,
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained") or p["bf16_tflops"], source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def swa_pairs(T: int, W: int) -> int:
    """Visible (query, key) pairs of one head: sum_i min(i + 1, W)."""
    if T <= W:
        return T * (T + 1) // 2
    return W * (W + 1) // 2 + (T - W) * W


def causal_pairs(T: int) -> int:
    return T * (T + 1) // 2


def algorithmic_work(op, s, pos=None):
    """(bound, amount, unit) of one call: compulsory HBM bytes for the
    bandwidth-bound calls, useful tensor FLOPs (visible pairs only) for the
    full causal ones.  Forward: 2 contractions (QK^T, PV) = 4 D FLOPs per
    pair; backward: 4 (dV, dP, dQ, dK) = 8 D, recomputation not counted."""
    tok, e = s.B * s.T, 2
    qb, kb = s.Hq * s.D * e, s.Hkv * s.D * e       # bytes per token of a q-like / k-like tensor
    if op == "gswa_fwd":      # read q, k, v, g; write y, lse
        return "hbm", tok * (3 * qb + 2 * kb + s.Hq * 4), "GB/s"
    if op == "gswa_bwd":      # read q, k, v, g, y, dy, lse; write dq, dk, dv, dg
        return "hbm", tok * (4 * qb + 2 * kb + s.Hq * 4 + 2 * qb + 2 * kb), "GB/s"
    if op == "full_attn_fwd":
        return "tensor", 4 * s.D * s.B * s.Hq * causal_pairs(s.T), "TFLOP/s"
    if op == "full_attn_bwd":
        return "tensor", 8 * s.D * s.B * s.Hq * causal_pairs(s.T), "TFLOP/s"
    if op == "gswa_decode":   # ring K/V of the visible slots + new q, k, v, g, y
        vis = min(pos + 1, s.window)
        return "hbm", s.B * (2 * s.Hkv * vis * s.D * e + 3 * s.Hq * s.D * e + 2 * s.Hkv * s.D * e), "GB/s"
    if op == "full_decode":   # K/V rows 0..pos + new q, k, v, y
        return "hbm", s.B * (2 * s.Hkv * (pos + 1) * s.D * e + 2 * s.Hq * s.D * e + 2 * s.Hkv * s.D * e), "GB/s"
    raise ValueError(op)


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region.

    Reads NVML every ~2 ms from a thread (read-only queries; no setting is
    touched); falls back to `nvidia-smi -lms 100` when NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []      # (sm_mhz, max_mhz, reasons)
        self.stop = threading.Event()
        self.thread = None
        self.smi = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def _poll(self, nv, h):
        masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), [n for n, m in masks if bits & m]))
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
        except Exception:
            try:
                self.smi = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.dev}",
                     "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                     "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                     "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.smi = None
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.smi is not None:
            self.smi.terminate()
            out, _ = self.smi.communicate(timeout=10)
            names = [n for n, _ in self.REASONS]
            for ln in out.splitlines():
                parts = [x.strip() for x in ln.split(",")]
                try:
                    self.samples.append((float(parts[0]), float(parts[1]),
                                         [n for n, v in zip(names, parts[2:6]) if v.lower() == "active"]))
                except (ValueError, IndexError):
                    continue

    def summary(self):
        if not self.samples:
            return None
        sm = [s[0] for s in self.samples]
        reasons = sorted({r for s in self.samples for r in s[2]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.samples[-1][1],
                "reasons": reasons, "samples": len(sm)}


# --------------------------------------------------------------------- workloads
class Step:
    """One step of a workload: `calls` is the ordered list of (entry point,
    callable); `h2d` / `d2h` map device tensors to pinned host copies for the
    end-to-end variant."""

    def __init__(self, name, s, tokens, calls, h2d, d2h, pos=None):
        self.name, self.s, self.tokens, self.calls = name, s, tokens, calls
        self.h2d, self.d2h, self.pos = h2d, d2h, pos

    def ops(self):
        seen = []
        for op, _ in self.calls:
            if op not in seen:
                seen.append(op)
        return seen

    def launches(self):
        return sum(LAUNCHES[op] for op, _ in self.calls)


def _ws(gca, op, shape, dev):
    n = gca.workspace_bytes(op, shape)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=dev)


def build_train(s, dev, seed):
    """One layer at training shape: gated-SWA fwd+bwd and full causal fwd+bwd on the same tensors."""
    import global_causal_attention_b200 as gca
    x = workloads.attention_inputs(s, seed, device=dev, with_grad=True)
    kw = dict(rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale)
    sh_swa = gca.make_shape(s.B, s.T, s.Hq, s.Hkv, s.D, s.window, **kw)
    sh_full = gca.make_shape(s.B, s.T, s.Hq, s.Hkv, s.D, 0, **kw)
    e = lambda t: torch.empty_like(t)
    f32 = lambda *shape: torch.empty(*shape, dtype=torch.float32, device=dev)
    y_s, y_f = e(x["q"]), e(x["q"])
    lse_s, lse_f = f32(s.B, s.Hq, s.T), f32(s.B, s.Hq, s.T)
    g_s = (e(x["q"]), e(x["k"]), e(x["k"]), e(x["q"]), f32(s.D), f32(s.D))
    g_f = (e(x["q"]), e(x["k"]), e(x["k"]), f32(s.D), f32(s.D))
    ws_sf = _ws(gca, gca.OP_GSWA_FWD, sh_swa, dev)
    ws_sb = _ws(gca, gca.OP_GSWA_BWD, sh_swa, dev)
    ws_ff = _ws(gca, gca.OP_FULL_FWD, sh_full, dev)
    ws_fb = _ws(gca, gca.OP_FULL_BWD, sh_full, dev)
    q, k, v, g, wq, wk, dy = (x[n] for n in ("q", "k", "v", "g", "wq", "wk", "dy"))
    calls = [
        ("gswa_fwd", lambda: gca.gswa_fwd(q, k, v, g, wq, wk, window=s.window, y=y_s, lse=lse_s, workspace=ws_sf,
                                          **kw)),
        ("gswa_bwd", lambda: gca.gswa_bwd(q, k, v, g, wq, wk, y_s, lse_s, dy, window=s.window, workspace=ws_sb,
                                          out=g_s, **kw)),
        ("full_attn_fwd", lambda: gca.full_attn_fwd(q, k, v, wq, wk, y=y_f, lse=lse_f, workspace=ws_ff, **kw)),
        ("full_attn_bwd", lambda: gca.full_attn_bwd(q, k, v, wq, wk, y_f, lse_f, dy, workspace=ws_fb, out=g_f,
                                                    **kw)),
    ]
    outs = [y_s, y_f, *g_s, *g_f]
    return Step("train_4k", s, s.B * s.T, calls, x, outs)


def build_prefill(name, s, dev, seed):
    """The 32-layer attention stack, forward, every layer on the same tensors
    (27 gated-SWA layers and 5 global layers, the schedule of the stack driver)."""
    from global_causal_attention_b200.stack import AttentionStack
    x = workloads.attention_inputs(s, seed, device=dev)
    st = AttentionStack(n_layers=LAYERS, window=s.window, rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps,
                        scale=s.scale)
    y_s, y_f = torch.empty_like(x["q"]), torch.empty_like(x["q"])
    lse = torch.empty(s.B, s.Hq, s.T, dtype=torch.float32, device=dev)
    outs = [(y_f, lse) if st.is_global(l) else (y_s, lse) for l in range(1, LAYERS + 1)]
    ws = st.prefill_workspace(s.B, s.T, s.Hq, s.Hkv, dev)
    calls = st.prefill_calls(x, outs, workspace=ws)
    return Step(name, s, s.B * s.T, calls, x, [y_s])


def build_decode(dev, seed):
    """One decode step of 32 sequences through the 32-layer stack.  The five
    global layers read one 262,144-token linear cache (34 GB of K/V; five
    distinct caches would not fit in HBM, and a cache this size streams from
    HBM either way); every SWA layer has its own 128-slot ring."""
    from global_causal_attention_b200.stack import AttentionStack
    d = workloads.DECODE_256K
    B, Hq, Hkv, D, W, Tmax = d["B"], d["Hq"], d["Hkv"], d["D"], d["window"], d["Tmax"]
    s = workloads.Shape(B=B, T=1, Hq=Hq, Hkv=Hkv, window=W, rope_base=d["rope_base"])
    st = AttentionStack(n_layers=LAYERS, window=W, rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps,
                        scale=s.scale)
    bf = dict(dtype=torch.bfloat16, device=dev)
    kc = workloads.fill_randn_bf16_(torch.empty(B, Hkv, Tmax, D, **bf), seed * 100 + 1)
    vc = workloads.fill_randn_bf16_(torch.empty(B, Hkv, Tmax, D, **bf), seed * 100 + 2)
    pos = torch.full((B,), d["pos"], dtype=torch.int64, device=dev)
    wq = torch.ones(D, **bf)
    wk = torch.ones(D, **bf)
    ins, caches, outs, h2d = [], [], [], {"pos": pos}
    for layer in range(1, LAYERS + 1):
        li = workloads.decode_inputs(B, Hq, Hkv, D, 1, seed=seed * 64 + layer, device=dev)
        x = {n: li[n] for n in ("q", "k", "v", "g")}
        x.update(wq=wq, wk=wk)
        for n in ("q", "k", "v", "g"):
            h2d[f"{n}{layer}"] = li[n]
        ins.append(x)
        outs.append(torch.empty_like(li["q"]))
        if st.is_global(layer):
            caches.append((kc, vc))
        else:
            caches.append((workloads.fill_randn_bf16_(torch.empty(B, Hkv, W, D, **bf), seed * 100 + 10 + layer),
                           workloads.fill_randn_bf16_(torch.empty(B, Hkv, W, D, **bf), seed * 100 + 50 + layer)))
    ws = st.decode_workspace(B, Hq, Hkv, Tmax, dev)
    calls = st.decode_calls(ins, caches, pos, outs, workspace=ws)
    return Step("decode_256k", s, B, calls, h2d, [outs[-1]], pos=d["pos"])


def build(name, dev, seed):
    if name == "train_4k":
        return build_train(WORKLOADS["train_4k"], dev, seed)
    if name in ("prefill_64k", "prefill_256k"):
        return build_prefill(name, WORKLOADS[name], dev, seed)
    if name == "decode_256k":
        return build_decode(dev, seed)
    raise ValueError(name)


# ---------------------------------------------------------------------- timing
def time_steps(step, K, W, stream, dist_on, sampler=None, per_op=False):
    """Device time of K steps after W warm-up steps (ms, max over ranks) and,
    with per_op, the summed device time of each entry point over the K steps,
    from CUDA events recorded around every call on the launching stream."""
    def run_one(evs=None):
        for i, (op, fn) in enumerate(step.calls):
            if evs is not None:
                evs[2 * i].record(stream)
            fn()
            if evs is not None:
                evs[2 * i + 1].record(stream)

    for _ in range(W):
        run_one()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(step.calls))] for _ in range(K)] \
        if per_op else [None] * K
    if sampler is not None:
        sampler.__enter__()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for kk in range(K):
        run_one(evsets[kk])
    e1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.__exit__(None, None, None)
    if dist_on:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    op_ms = {}
    if per_op:
        for evs in evsets:
            for i, (op, _) in enumerate(step.calls):
                op_ms[op] = op_ms.get(op, 0.0) + evs[2 * i].elapsed_time(evs[2 * i + 1])
    if dist_on:
        ms = max_over_ranks(ms, "cuda")
    return ms, op_ms


def max_over_ranks(ms, device):
    """The slowest rank's time: every rank contributes its own and gets the max."""
    t = torch.tensor([float(ms)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_e2e(steps, host_in, host_out, K, W, stream, dist_on):
    """Device time of K end-to-end steps (ms, max over ranks) after W warm-up
    steps.  Step i uses buffer set i % 2: its inputs are copied in on an
    upload stream (once the compute of step i - 2 is done with the set), it
    runs on `stream`, and its outputs are copied out on a download stream, so
    the copies of neighbouring steps overlap this step's compute.  The timed
    region starts before the first upload and ends after the last download."""
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    done = [torch.cuda.Event(), torch.cuda.Event()]      # compute of the set's last step finished
    loaded = [torch.cuda.Event(), torch.cuda.Event()]    # the set's inputs are on the device
    freed = [torch.cuda.Event(), torch.cuda.Event()]     # the set's outputs are on the host

    def run(n_steps):
        for i in range(n_steps):
            st = steps[i % 2]
            slot = i % 2
            up.wait_event(freed[slot])   # a never-recorded event is already complete
            with torch.cuda.stream(up):
                for name, t in host_in.items():
                    st.h2d[name].copy_(t, non_blocking=True)
                loaded[slot].record(up)
            stream.wait_event(loaded[slot])
            for _, fn in st.calls:
                fn()
            done[slot].record(stream)
            down.wait_event(done[slot])
            with torch.cuda.stream(down):
                for h, t in zip(host_out[slot], st.d2h):
                    h.copy_(t, non_blocking=True)
                freed[slot].record(down)

    run(W)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    run(K)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist_on:
        torch.distributed.barrier()
        ms = max_over_ranks(ms, "cuda")
    return ms


def tensor_peak(pk, clocks, timed_s):
    """(peak TFLOP/s, which) for the tensor-bound entry points of this run: the
    burst peak (cuBLAS measured in isolation at full clocks) when the timed
    region is short (< 1 s) or ran at full clocks without the power cap, the
    sustained peak (cuBLAS in a seconds-long loop under the power cap)
    otherwise."""
    full_clock = clocks is not None and clocks["sm_mhz"] >= 0.98 * clocks["sm_max_mhz"]
    capped = clocks is not None and "sw_power_cap" in clocks["reasons"]
    if timed_s < 1.0 or (full_clock and not capped):
        return pk["bf16_tflops"], "burst"
    return pk["bf16_tflops_sustained"], "sustained"


def op_table(step, op_ms, K, pk, tpeak):
    """Per entry point: calls per step, ms per call, achieved rate against its
    bound.  Tensor-bound calls carry the fraction of both tensor peaks."""
    table = {}
    for op in step.ops():
        n = sum(1 for o, _ in step.calls if o == op)
        per_call = op_ms[op] / (K * n)
        bound, amount, unit = algorithmic_work(op, step.s, step.pos)
        e = {"calls_per_step": n, "ms_per_call": per_call, "bound": bound, "unit": unit,
             "algorithmic_per_call": amount, "launches_per_call": LAUNCHES[op]}
        if bound == "hbm":
            achieved = amount / (per_call / 1e3) / 1e9
            e.update(achieved=achieved, peak=pk["hbm_gbs"], frac=achieved / pk["hbm_gbs"])
        else:
            achieved = amount / (per_call / 1e3) / 1e12
            e.update(achieved=achieved, peak=tpeak[0], peak_kind=tpeak[1], frac=achieved / tpeak[0],
                     frac_burst=achieved / pk["bf16_tflops"],
                     frac_sustained=achieved / pk["bf16_tflops_sustained"])
        table[op] = e
    return table


# ---------------------------------------------------------------- the oracle
def _oracle_cores():
    import oracle
    return oracle.num_threads()


_ORACLE_INPUTS = {}


def _memo(key, make):
    """Oracle inputs are generated once per process (a 262,144-token cache takes seconds)."""
    if key not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[key] = make()
    return _ORACLE_INPUTS[key]


def oracle_sample(name, budget_s):
    """Run the float64 oracle on a bounded sample of one step of `name` and
    extrapolate to the whole step.  Returns (measured s, extrapolated s for one
    full step, threads used, description)."""
    import oracle
    cores = _oracle_cores()
    if name == "train_4k":
        s = WORKLOADS["train_4k"]
        # one sequence's causal prefix of T' tokens over G KV groups: the outputs of a
        # prefix depend on the prefix only, so this is an exact slice of the step.
        # G covers every host core the oracle can use (it runs the KV groups on
        # separate threads); the prefix shrinks to fit the budget: with one
        # group per thread the whole 4,096-token prefix takes about 20 s, the
        # full causal part (most of it) growing as T'^2.
        G = max(1, min(s.Hkv, cores))
        Tp = s.T if budget_s >= 20.0 else max(128, int(s.T * math.sqrt(budget_s / 20.0)) // 128 * 128)
        sg = s.replace(B=1, T=Tp, Hq=4 * G, Hkv=G)
        x = _memo(("train", Tp, G), lambda: workloads.attention_inputs(sg, 0, with_grad=True))
        kw = oracle.shape_kwargs(sg)
        t0 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window, gated=True, **kw)
        oracle.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], x["dy"], window=s.window, gated=True,
                        **kw)
        t1 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False, **kw)
        oracle.attn_bwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], x["dy"], window=0, gated=False, **kw)
        t2 = time.perf_counter()
        groups = s.B * s.Hkv / G
        full = (t1 - t0) * groups * swa_pairs(s.T, s.window) / swa_pairs(Tp, s.window) + \
               (t2 - t1) * groups * causal_pairs(s.T) / causal_pairs(Tp)
        desc = (f"gated-SWA fwd+bwd and full causal fwd+bwd of the first {Tp} tokens of 1 sequence x {G} of "
                f"{s.Hkv} KV groups ({4 * G} query heads), float64; extrapolated to {s.B}x{s.T}x{s.Hq} heads "
                f"by the exact visible-pair counts of each part")
        return t2 - t0, full, min(G, cores), desc
    if name in ("prefill_64k", "prefill_256k"):
        s = WORKLOADS[name]
        # about 0.1 s of oracle work per sampled row at 64K (rows cost in proportion to position)
        nrows = max(2, min(256, int(budget_s / (0.12 * s.T / 65536))))
        rows = workloads.sample_rows(s.T, nrows, seed=3).numpy()
        G = min(s.Hkv, cores)
        sg = s.replace(B=1, Hq=4 * G, Hkv=G)
        x = _memo((name, G), lambda: workloads.attention_inputs(sg, 0))
        kw = oracle.shape_kwargs(sg)
        t0 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window, gated=True,
                        rows=rows, **kw)
        t1 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], None, x["wq"], x["wk"], window=0, gated=False, rows=rows, **kw)
        t2 = time.perf_counter()
        groups = s.B * s.Hkv / G
        n_swa = sum(1 for l in range(1, LAYERS + 1) if not workloads.layer_is_global(l))
        n_full = LAYERS - n_swa
        ps = sum(min(int(i) + 1, s.window) for i in rows)
        pf = sum(int(i) + 1 for i in rows)
        full = n_swa * (t1 - t0) * groups * swa_pairs(s.T, s.window) / ps + \
               n_full * (t2 - t1) * groups * causal_pairs(s.T) / pf
        desc = (f"gated-SWA and full causal forward of {len(rows)} seeded query positions of 1 sequence x {G} KV "
                f"groups ({4 * G} query heads) at T={s.T}, float64; extrapolated to the {n_swa}+{n_full}-layer "
                f"stack by the exact visible-pair counts (the per-call key preparation is not scaled)")
        return t2 - t0, full, min(G, cores), desc
    if name == "decode_256k":
        d = workloads.DECODE_256K
        s = workloads.Shape(B=1, T=1, Hq=d["Hq"], Hkv=d["Hkv"], window=d["window"], rope_base=d["rope_base"])
        kw = oracle.shape_kwargs(s)
        xs = _memo("ring", lambda: workloads.decode_inputs(1, d["Hq"], d["Hkv"], d["D"], d["window"], seed=0))
        pos = [d["pos"]]
        xf = _memo("linear", lambda: workloads.decode_inputs(1, d["Hq"], d["Hkv"], d["D"], d["Tmax"], seed=0))
        reps = max(1, min(d["B"], int(budget_s / 0.4)))   # about 0.4 s per repetition
        t_swa = t_full = 0.0
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle.decode(xs["q"], xs["k"], xs["v"], xs["g"], xs["wq"], xs["wk"], xs["k_cache"], xs["v_cache"],
                          pos, window=d["window"], gated=True, **kw)
            t1 = time.perf_counter()
            oracle.decode(xf["q"], xf["k"], xf["v"], None, xf["wq"], xf["wk"], xf["k_cache"], xf["v_cache"],
                          pos, window=0, gated=False, **kw)
            t2 = time.perf_counter()
            t_swa += t1 - t0
            t_full += t2 - t1
        n_full = sum(1 for l in range(1, LAYERS + 1) if workloads.layer_is_global(l))
        full = d["B"] * ((LAYERS - n_full) * t_swa + n_full * t_full) / reps
        desc = (f"{reps} x (one SWA-layer ring decode and one global-layer 262,144-token-cache decode) of one "
                f"sequence, float64; extrapolated to {d['B']} sequences and the 27+5-layer stack")
        return t_swa + t_full, full, min(d["Hkv"], cores), desc
    raise ValueError(name)


def cpu_baseline(name, tokens):
    measured, full, cores, desc = oracle_sample(name, budget_s=15.0)
    return {"value": tokens / full, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{desc}; {measured:.1f} s measured"}


def run_reference(args):
    """--impl reference: the oracle, timed on the host cores, same metric and config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = 120.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        oracle_sample(args.workload, budget)
    measured = extrap = 0.0
    desc, cores = "", 1
    for _ in range(args.steps):
        m, e, cores, desc = oracle_sample(args.workload, budget)
        measured += m
        extrap += e
    tokens = tokens_per_step(args.workload)
    value = tokens * args.steps / extrap
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": extrap * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}; {measured:.1f} s measured over {args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def tokens_per_step(name):
    if name == "decode_256k":
        return workloads.DECODE_256K["B"]
    s = WORKLOADS[name]
    return s.B * s.T


def workload_config(name, n):
    if name == "decode_256k":
        d = workloads.DECODE_256K
        return {"workload": f"decode_256k: one decode step of {d['B']} sequences at position {d['pos']} through "
                            f"the 32-layer stack (27 gswa_decode on 128-slot rings + 5 full_decode on a "
                            f"{d['Tmax']}-token linear cache), {d['Hq']}q/{d['Hkv']}kv D{d['D']}, base "
                            f"{d['rope_base']:g}",
                "global_batch": d["B"] * n, "seq_len": d["Tmax"], "parallelism": f"replicas x{n} (weak)",
                "l2": "caches larger than L2 (no flush needed)"}
    s = WORKLOADS[name]
    what = ("gswa_fwd + gswa_bwd + full_attn_fwd + full_attn_bwd on the same tensors" if name == "train_4k"
            else "32-layer stack forward: 27 gswa_fwd + 5 full_attn_fwd (layers 6, 12, 18, 24, 30)")
    return {"workload": f"{name}: {what} (B{s.B} T{s.T} {s.Hq}q/{s.Hkv}kv D{s.D} W{s.window} "
                        f"rope {s.rope_dims}/{s.D} base {s.rope_base:g})",
            "global_batch": s.B * n, "seq_len": s.T, "parallelism": f"replicas x{n} (weak)",
            "l2": "inputs larger than L2 (no flush needed)"}


DEFAULT_STEPS = {"train_4k": 100, "prefill_64k": 5, "prefill_256k": 2, "decode_256k": 30}
# Steps of the other workloads that a default (train_4k) run also times.
EXTRA_STEPS = {"prefill_64k": 4, "prefill_256k": 2, "decode_256k": 20}
EXTRA_WARMUP = {"prefill_64k": 3, "prefill_256k": 3, "decode_256k": 3}


def measure(name, dev, seed, steps, warmup, stream, dist_on, pk):
    """Build workload `name`, time `steps` steps after `warmup` (clocks sampled),
    and return (step, ms, clocks, per-entry-point table, roofline of the
    dominant entry point)."""
    import global_causal_attention_b200 as gca
    step = build(name, dev, seed=seed)
    clk = ClockSampler(torch.cuda.current_device())
    ms, op_ms = time_steps(step, steps, warmup, stream, dist_on, sampler=clk, per_op=True)
    clocks = clk.summary()
    if gca.gswa_check_status() != 0:
        raise RuntimeError("device status reports a timed-out wait or a bad position")
    tpeak = tensor_peak(pk, clocks, ms / 1e3)
    ops = op_table(step, op_ms, steps, pk, tpeak)
    for o in ops:
        ops[o]["traffic"] = TRAFFIC.get((name, o))
    dom = max(ops, key=lambda o: ops[o]["ms_per_call"] * ops[o]["calls_per_step"])
    d = ops[dom]
    roofline = {"bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
                "frac": d["frac"], "traffic": d["traffic"], "kernel": dom,
                "launches": d["launches_per_call"], "ms_per_launch": d["ms_per_call"],
                "algorithmic_per_launch": d["algorithmic_per_call"],
                "peak_source": pk["source"] + (f" {d['peak_kind']}" if d["bound"] == "tensor" else "")}
    if d["bound"] == "tensor":
        roofline["frac_burst"] = d["frac_burst"]
        roofline["frac_sustained"] = d["frac_sustained"]
    return step, ms, clocks, ops, roofline


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="train_4k", choices=WORKLOAD_NAMES)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads' device timings that the default train_4k run adds")
    ap.add_argument("--batch", type=int, default=None,
                    help="run the workload at this many sequences instead of its own batch (a smaller case "
                         "for profiler captures; the JSON line's config reports the batch used)")
    args = ap.parse_args()
    if args.batch is not None:
        import dataclasses
        WORKLOADS[args.workload] = dataclasses.replace(WORKLOADS[args.workload], B=args.batch)
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    import global_causal_attention_b200 as gca
    gca.lib()
    pk = peaks()
    stream = torch.cuda.current_stream(dev)
    step, ms, clocks, ops, roofline = measure(args.workload, dev, rank, args.steps, args.warmup, stream, dist_on,
                                              pk)
    tokens = step.tokens * world
    value = tokens * args.steps / (ms / 1e3)

    # End to end through the public API: every step's inputs copied from pinned
    # host memory to the device and its outputs back to pinned host memory,
    # pipelined like a data loader (two device copies of the step's buffers).
    host_in = {n: t.to("cpu").pin_memory() for n, t in step.h2d.items()}
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in step.d2h] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    step2 = build(args.workload, dev, seed=rank)
    e2e_k = max(3, min(args.steps, 8))
    e2e_ms = time_e2e([step, step2], host_in, host_out, e2e_k, 2, stream, dist_on)
    del step2
    e2e_value = tokens * e2e_k / (e2e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, step.tokens)

    # The other workloads, timed the same way in the same run (one GPU only):
    # their device time, per-entry-point table and roofline.
    launches = step.launches() * args.steps
    extra = None
    if world == 1 and args.workload == "train_4k" and not args.no_extra:
        del step, host_in, host_out
        extra = {}
        for name in WORKLOAD_NAMES:
            if name == args.workload:
                continue
            torch.cuda.empty_cache()
            st2, ms2, clk2, ops2, roof2 = measure(name, dev, rank, EXTRA_STEPS[name], EXTRA_WARMUP[name], stream,
                                                  False, pk)
            extra[name] = {"steps": EXTRA_STEPS[name], "warmup": EXTRA_WARMUP[name],
                           "ms_per_step": ms2 / EXTRA_STEPS[name],
                           "value": st2.tokens * EXTRA_STEPS[name] / (ms2 / 1e3), "unit": UNIT,
                           "config": workload_config(name, 1)["workload"], "roofline": roof2, "ops": ops2,
                           "gpu_launches": st2.launches() * EXTRA_STEPS[name], "clocks": clk2}
            del st2
        if gca.gswa_check_status() != 0:
            raise RuntimeError("device status reports a timed-out wait or a bad position")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args.workload, world),
            "roofline": roofline,
            "ops": ops,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if extra is not None:
            line["workloads"] = extra
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
