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

# Hot-path kernels each workload's step runs, in order.
STEP_OPS = {
    "train_4k": ["gswa_fwd"],
    "prefill_64k": ["gswa_fwd"],
    "prefill_256k": ["gswa_fwd"],
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def swa_fwd_bytes(s) -> int:
    """Compulsory HBM bytes of one gated-SWA forward: read q, k, v, g; write y, lse."""
    tok = s.B * s.T
    return tok * (s.Hq * s.D * 2 * 3 + s.Hkv * s.D * 2 * 2 + s.Hq * 4)


def swa_pairs(T: int, W: int) -> int:
    """Visible (query, key) pairs of one head: sum_i min(i + 1, W)."""
    if T <= W:
        return T * (T + 1) // 2
    return W * (W + 1) // 2 + (T - W) * W


def swa_fwd_flops(s) -> int:
    """Algorithmic FLOPs of the two contractions over the unmasked pairs."""
    return 4 * s.B * s.Hq * s.D * swa_pairs(s.T, s.window)


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


def make_step(ops, s, x, dev):
    """Device buffers + a callable running one step; returns (step, outputs, n_launches)."""
    import global_causal_attention_b200 as gca
    y = torch.empty_like(x["q"])
    lse = torch.empty((s.B, s.Hq, s.T), dtype=torch.float32, device=dev)

    def step():
        for op in ops:
            if op == "gswa_fwd":
                gca.gswa_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                             rope_dims=s.rope_dims, rope_base=s.rope_base, eps=s.eps, scale=s.scale,
                             y=y, lse=lse)
            else:
                raise ValueError(op)

    return step, {"y": y, "lse": lse}, len(ops)


def time_steps(step, K, W, stream, dist_on, sampler=None):
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.__enter__()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.__exit__(None, None, None)
    if dist_on:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    if dist_on:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return ms


def launch_ms(fn, reps, stream):
    """Average duration of one launch of `fn`, CUDA events on its stream."""
    fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def cpu_baseline(s, target_s=15.0):
    """The float64 oracle on a bounded sample of the workload's query rows."""
    import oracle
    from workloads import attention_inputs, sample_rows
    x = attention_inputs(s, 0)
    nrows = 8
    spent = 0.0
    while True:
        rows = sample_rows(s.T, nrows, seed=3).numpy()
        t0 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                        gated=True, rows=rows, **oracle.shape_kwargs(s))
        spent = time.perf_counter() - t0
        if spent * 2 > target_s or nrows >= s.T:
            break
        nrows = min(s.T, nrows * max(2, int(target_s / max(spent, 1e-3) / 2)))
    tokens = s.B * len(rows)
    return {"value": tokens / spent, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"gated-SWA forward of {len(rows)} seeded query positions x {s.B} sequences "
                      f"x all {s.Hq} heads of {s.B}x{s.T} (keys prepared for every position), "
                      f"float64, {spent:.1f} s"}


def run_reference(args):
    """--impl reference: the oracle, timed on the host cores, same metric/config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = WORKLOADS[args.workload]
    import oracle
    from workloads import attention_inputs, sample_rows
    x = attention_inputs(s, 0)
    rows = sample_rows(s.T, 16, seed=3).numpy()
    kw = oracle.shape_kwargs(s)

    def step():
        oracle.attn_fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=s.window,
                        gated=True, rows=rows, **kw)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    tokens = s.B * len(rows) * args.steps
    value = tokens / dt
    sample = (f"gated-SWA forward of {len(rows)} seeded query positions x {s.B} sequences x all "
              f"{s.Hq} heads of {s.B}x{s.T} per step, float64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(s, args.workload, STEP_OPS[args.workload], args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(s, name, ops, n):
    return {"workload": f"{name}: " + " + ".join(ops) + f" (B{s.B} T{s.T} {s.Hq}q/{s.Hkv}kv "
                        f"D{s.D} W{s.window} rope {s.rope_dims}/{s.D} base {s.rope_base:g})",
            "global_batch": s.B * n, "seq_len": s.T, "parallelism": f"replicas x{n} (weak)",
            "l2": "inputs larger than L2 (no flush needed)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="train_4k", choices=sorted(STEP_OPS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
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
    s = WORKLOADS[args.workload]
    ops = STEP_OPS[args.workload]
    x = workloads.attention_inputs(s, seed=rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    step, outs, launches_per_step = make_step(ops, s, x, dev)

    clk = ClockSampler(torch.cuda.current_device())
    ms = time_steps(step, args.steps, args.warmup, stream, dist_on, sampler=clk)
    clocks = clk.summary()
    if gca.gswa_check_status() != 0:
        raise RuntimeError("device status reports a timed-out wait")
    tokens_per_step = s.B * s.T * world
    value = tokens_per_step * args.steps / (ms / 1e3)

    # Roofline of the dominant kernel (the gated-SWA forward: HBM-bound).
    pk = peaks()
    fwd_ms = launch_ms(step, 10, stream)
    fwd_bytes = swa_fwd_bytes(s)
    achieved = fwd_bytes / (fwd_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": "gswa_fwd", "achieved": achieved, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None,
                "algorithmic_bytes_per_launch": fwd_bytes, "launch_ms": fwd_ms,
                "peak_source": pk["source"], "tensor_tflops": swa_fwd_flops(s) / (fwd_ms / 1e3) / 1e12}

    # End to end through the public API: pinned host inputs -> device, step,
    # output back to the host, every step.
    host = {n: t.to("cpu").pin_memory() for n, t in x.items()}
    y_host = torch.empty(outs["y"].shape, dtype=outs["y"].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = y_host.numel() * y_host.element_size()

    def e2e_step():
        for n, t in host.items():
            x[n].copy_(t, non_blocking=True)
        step()
        y_host.copy_(outs["y"], non_blocking=True)

    e2e_steps = max(2, min(args.steps, 5))
    e2e_ms = time_steps(e2e_step, e2e_steps, 1, stream, dist_on)
    e2e_value = tokens_per_step * e2e_steps / (e2e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(s)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(s, args.workload, ops, world),
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
