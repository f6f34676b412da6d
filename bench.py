"""Benchmark of the sharded gated MLP on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one forward pass of the SwiGLU MLP of the Llama-3-8B shape
(n=4096 tokens, d_model=4096, d_ff=14336, P=8 logical weight shards, bf16
with fp32 accumulation) through the C ABI: gate/up projection with the fused
activation, then the row-split down projection accumulated in place, shard
chunk after shard chunk.  Other workloads (--workload) are for ad-hoc
measurements; the default is the one the headline metric is quoted on.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, timed with CUDA events on the
launching stream; the max over ranks is reported.  The weights alone (352 MB)
exceed the 126 MB L2, so no flush is needed between steps.  Under torchrun
(N > 1) every rank runs an independent replica (the path has no
cross-device step), so scaling is weak and value = N x per-step FLOPs / max
time.

--impl reference times the fp64 CPU oracle on a bounded sample of token rows
of the same workload (rank 0 only; other ranks exit at once).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import (ATTN_WORKLOADS, LLAMA8B, WORKLOADS, make_attn_inputs,  # noqa: E402
                       make_inputs)

PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# the csrc headers each kernel is built from (a change to any of them voids its
# committed ncu traffic figure)
FORWARD_SOURCES = ["ptx.cuh", "pipeline.cuh", "pipeline2.cuh", "recipes.cuh"]


def kernel_sources(kernel: str) -> list[str]:
    if kernel.endswith("_save") or kernel.startswith("bwd_dh_factor"):
        return FORWARD_SOURCES + ["bwd_pair.cuh", "train_pair.cuh"]
    if kernel.startswith("dgrad_wgrad"):
        return FORWARD_SOURCES + ["bwd_pair.cuh", "train_pair.cuh", "grad_pair.cuh"]
    if kernel.startswith("fused_fwd"):
        return FORWARD_SOURCES + ["fused.cuh"]
    if kernel.startswith("fused_passes"):
        return FORWARD_SOURCES + ["fused.cuh", "fused2.cuh"]
    if kernel.startswith(("bwd_", "wgrad_")):
        return FORWARD_SOURCES + ["bwd_pair.cuh"]
    if kernel.startswith("f32_"):
        return ["simt_f32.cuh"]
    if kernel.startswith("attn_core"):
        return ["ptx.cuh", "pipeline.cuh", "attn.cuh"]
    return FORWARD_SOURCES


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {"bf16_tflops": j["bf16_tflops"], "bf16_tflops_sustained": j["bf16_tflops_sustained"],
                "hbm_gbs": j["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "source": "fallback"}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in kernel_sources(kernel):
        with open(os.path.join(ROOT, "sequence_transformer_mlp_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, wl_name: str, launches_per_step: int):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when there is none for this workload or the kernel sources changed since."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as fh:
        j = json.load(fh)
    ent = j.get(wl_name, {}).get(kernel)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled DURING the timed region.

    In-process NVML queries (read-only) from a background thread every few
    milliseconds, so that even a timed region of a few tens of milliseconds
    holds samples; ``nvidia-smi -lms 200`` in a subprocess when NVML is not
    importable.  Nothing here changes a GPU setting."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.004
    # clock-event reason bits (NVML): power capping, and the slowdowns that void a timing
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        try:
            self.uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
        except Exception:  # pragma: no cover
            self.uuid = None
        self.gpu_index = gpu_index
        self.rows = []     # (time.time(), sm_mhz, max_mhz, power_w, reasons bitmask)
        self.t0 = self.t1 = None
        self.mode = None
        self.proc = self.thread = None
        self.path = None

    # ---------------------------------------------------------------- NVML thread
    def _nvml_start(self):
        import threading
        import pynvml as nv
        nv.nvmlInit()
        try:
            h = nv.nvmlDeviceGetHandleByUUID(("GPU-" + self.uuid) if self.uuid else "")
        except Exception:
            h = nv.nvmlDeviceGetHandleByIndex(self.gpu_index)
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    rs = int(get_reasons(h)) if get_reasons else 0
                    self.rows.append((time.time(), float(sm), float(max_mhz), pw, rs))
                except Exception:  # pragma: no cover
                    pass
                self._stop.wait(self.PERIOD_S)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        self._nv = nv
        self.mode = "nvml"

    # ---------------------------------------------------------------- nvidia-smi fallback
    def _smi_start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.out = open(self.path, "w")
        sel = [f"--id=GPU-{self.uuid}"] if self.uuid else [f"--id={self.gpu_index}"]
        self.proc = subprocess.Popen(
            ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
             "-lms", "200"], stdout=self.out, stderr=subprocess.DEVNULL)
        self.mode = "nvidia-smi"

    def __enter__(self):
        try:
            self._nvml_start()
        except Exception:
            try:
                self._smi_start()
            except (OSError, FileNotFoundError):
                self.mode = None
        # wait for the first sample, so that sampling covers the timed region
        t_end = time.time() + 5.0
        while self.mode and time.time() < t_end and not self._have_sample():
            time.sleep(0.01)
        return self

    def _have_sample(self):
        if self.mode == "nvml":
            return bool(self.rows)
        return os.path.getsize(self.path) > 0

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        if self.mode == "nvml":
            self._stop.set()
            self.thread.join(timeout=2)
            try:
                self._nv.nvmlShutdown()
            except Exception:  # pragma: no cover
                pass
        elif self.mode == "nvidia-smi":
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()
            self._read_smi()

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    sm, mx, pw = float(parts[2]), float(parts[3]), float(parts[4])
                except ValueError:
                    continue
                rs = 0
                for i, nm in enumerate(names):
                    if parts[6 + i] == "Active":
                        rs |= self.REASON_BITS[nm]
                self.rows.append((ts, sm, mx, pw, rs))
        os.unlink(self.path)

    def summary(self):
        return summarise_clocks(self.rows, self.t0, self.t1, self.mode, self.REASON_BITS)


def summarise_clocks(rows, t0, t1, source, reason_bits):
    """Median SM clock, max clock, active reasons and power over the samples
    taken inside [t0, t1] (all samples when none fell inside)."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None,
                "reasons": ["no clock samples" if source else "no NVML or nvidia-smi"],
                "samples": 0, "samples_in_timed_region": 0, "source": source}
    window = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
    use = window or rows
    reasons = sorted({nm for r in use for nm, bit in reason_bits.items() if r[4] & bit})
    return {"sm_mhz": statistics.median(r[1] for r in use),
            "sm_max_mhz": max(r[2] for r in use),
            "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(window),
            "power_w_median": statistics.median(r[3] for r in use), "source": source}


def _np64(t):
    return None if t is None else t.double().numpy()


def oracle_sample(wl, inp, rows: int, cols: int) -> dict:
    """The fp64 oracle, as it stands, on a sample of one step of `wl`.

    Forward: the sharded block on the first `rows` token rows (a row of Y
    depends only on its own row of X).  Forward+backward adds the input
    gradient on the same rows and the weight gradients on the first `cols`
    hidden columns (column j of dW_gate / dW_up and row j of dW_down depend
    only on hidden unit j).  Returns the seconds of each part and the full
    step's CPU time extrapolated from them (per row, per column)."""
    import oracle
    A, B, Wu = _np64(inp["A"]), _np64(inp["B"]), _np64(inp["Wu"])
    X = _np64(inp["X"][:rows])
    t0 = time.perf_counter()
    oracle.mlp_sharded(X, A, Wu, B, wl.act, wl.P)
    parts = {"fwd_rows_s": time.perf_counter() - t0}
    full = parts["fwd_rows_s"] * wl.n / rows
    if wl.backward:
        dY = _np64(inp["dY"])
        t0 = time.perf_counter()
        oracle.mlp_backward(X, A, Wu, B, dY[:rows], wl.act, outputs=("dX",))
        parts["dx_rows_s"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.mlp_backward(_np64(inp["X"]), A[:, :cols], None if Wu is None else Wu[:, :cols],
                            B[:cols, :], dY, wl.act, outputs=("dA", "dWu", "dB"))
        parts["dw_cols_s"] = time.perf_counter() - t0
        full += parts["dx_rows_s"] * wl.n / rows + parts["dw_cols_s"] * wl.f / cols
    parts["extrapolated_full_step_s"] = full
    return parts


def _sample_text(wl, rows, cols, parts):
    txt = f"first {rows} token rows of {wl.name}: sharded forward"
    if wl.backward:
        txt += f" and input gradient; first {cols} hidden columns: weight gradients"
    txt += (f" (fp64 oracle, {sum(v for k, v in parts.items() if k.endswith('_s') and k != 'extrapolated_full_step_s'):.1f} s); "
            f"full step extrapolated per row / column: {parts['extrapolated_full_step_s']:.1f} s")
    return txt


def workload_flops(wl) -> float:
    return wl.flops_forward() + (wl.flops_backward() if wl.backward else 0)


def reference_arm(args, wl, rank):
    """fp64 CPU oracle on a bounded sample of the workload's step (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    inp = make_inputs(wl)
    want = args.ref_rows or (64 if wl.backward else 256)
    rows = max(1, min(wl.n, want))
    cols = max(1, min(wl.f, want))
    for _ in range(args.warmup):
        oracle_sample(wl, inp, rows, cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        parts = oracle_sample(wl, inp, rows, cols)
    dt = (time.perf_counter() - t0) / args.steps
    # the throughput of the oracle on the sample = the full step's FLOPs over
    # its extrapolated CPU time
    tflops = workload_flops(wl) / parts["extrapolated_full_step_s"] / 1e12
    line = {
        "impl": "reference", "metric": metric_name(wl), "value": tflops,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded torch.randn)",
        "tokens_per_s": wl.n / parts["extrapolated_full_step_s"],
        "config": {"workload": wl.name, "n_tokens": wl.n, "d_model": wl.d, "d_ff": wl.f,
                   "P": wl.P, "sample_rows": rows, **({"sample_cols": cols} if wl.backward else {})},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": _sample_text(wl, rows, cols, parts) + " per step",
                         "extrapolated_full_step_s": parts["extrapolated_full_step_s"]},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, target_s=12.0):
    """The oracle, as it stands, on a bounded sample of the step (rank 0, N = 1):
    about `target_s` seconds of CPU work, split between the step's parts."""
    import oracle
    inp = make_inputs(wl)
    probe = 16
    pp = oracle_sample(wl, inp, probe, probe)
    nparts = 3 if wl.backward else 1
    per = target_s / nparts
    row_s = pp["fwd_rows_s"] + pp.get("dx_rows_s", 0.0)
    rows = int(max(probe, min(wl.n, probe * per * (2 if wl.backward else 1) / max(row_s, 1e-9))))
    cols = int(max(probe, min(wl.f, probe * per / max(pp.get("dw_cols_s", 1.0), 1e-9))))
    parts = oracle_sample(wl, inp, rows, cols)
    full = parts["extrapolated_full_step_s"]
    return {"value": workload_flops(wl) / full / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": _sample_text(wl, rows, cols, parts) + f"; tokens/s {wl.n / full:.1f}",
            "extrapolated_full_step_s": full}


def metric_name(wl) -> str:
    return ("sharded gated-MLP forward TFLOP/s" if not wl.backward
            else "sharded gated-MLP forward+backward TFLOP/s")


def max_over_ranks(values, dist, device):
    """Element-wise maximum of `values` over all ranks (every rank gets it)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(world: int, flops_per_step: float, ms_max: float) -> float:
    """Whole-job TFLOP/s of `world` independent replicas timed by the slowest."""
    return world * flops_per_step / (ms_max * 1e-3) / 1e12


def end_to_end(args, inp, dev, step, Y, stream, barrier):
    """The same step through the public call with host buffers, pipelined as a
    serving loop would run it: every step copies its X in from pinned host
    memory (copy-in stream) and reads its Y back (copy-out stream), and the
    copies of neighbouring steps overlap the compute of the current one
    (device X and Y double-buffered, ordered with events).  All copies are
    inside the timed region.  Returns (ms per step, host X, host Y)."""
    n, d = inp["X"].shape
    Xh = inp["X"].pin_memory()
    Yh = [torch.empty(n, d, dtype=Y.dtype).pin_memory() for _ in range(2)]
    Xd = [torch.empty_like(dev["X"]) for _ in range(2)]
    Yd = [torch.empty_like(Y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(k):
        for i in range(k):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[b])      # X[b] of step i-2 consumed
                Xd[b].copy_(Xh, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])         # Y[b] of step i-2 read back
            step(Xd[b], Yd[b])
            comp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                Yh[b].copy_(Yd[b], non_blocking=True)
                out_done[b].record(s_out)

    run(4)
    torch.cuda.synchronize()
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(s_in)
    run(args.steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e3.record(s_out)
    torch.cuda.synchronize()
    barrier()
    return e2.elapsed_time(e3) / args.steps, Xh, Yh[0]


def setup_mlp(args, wl, T, stream):
    """The MLP step (forward, or forward+backward) through the C ABI."""
    inp = make_inputs(wl)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    n, d, f, P = wl.n, wl.d, wl.f, wl.P
    sched = args.sched or wl.sched
    dt = "f32" if wl.dtype == "f32" else "bf16"
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    Y = torch.empty(n, d, dtype=tdt, device="cuda")
    saved_act = wl.backward and not args.bwd_recompute
    if not wl.backward:
        need = T.tsp_mlp_workspace_size(n, d, f, P, wl.act, dt, sched)
    elif saved_act:
        need = T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, wl.act)
    else:
        need = T.tsp_mlp_workspace_size(n, d, f, P, wl.act, dt, sched, backward=True)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    st = {}
    if wl.backward:
        st["dX"] = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
        st["dWg"] = torch.empty(d, f, dtype=torch.float32, device="cuda")
        st["dWu"] = (torch.empty(d, f, dtype=torch.float32, device="cuda")
                     if wl.act == "swiglu" else None)
        st["dWd"] = torch.empty(f, d, dtype=torch.float32, device="cuda")
        if saved_act:
            # the training forward keeps H and the activation's factors for the backward
            st["n_saved"] = T.tsp_mlp_saved_size(n, d, f, P, wl.act)
            st["saved"] = torch.empty(st["n_saved"], dtype=torch.uint8, device="cuda")
        else:
            st["ws_f"] = torch.empty(
                max(T.tsp_mlp_workspace_size(n, d, f, P, wl.act, "bf16", sched), 1),
                dtype=torch.uint8, device="cuda")

    def step(x=dev["X"], y=Y):
        if saved_act:
            T.tsp_mlp_forward_train(x, dev["A"], dev["Wu"], dev["B"], n, d, f, P, wl.act, y,
                                    st["saved"], st["n_saved"], stream)
            T.tsp_mlp_backward_saved(x, dev["A"], dev["Wu"], dev["B"], dev["dY"], st["saved"],
                                     st["n_saved"], n, d, f, P, wl.act, st["dX"], st["dWg"],
                                     st["dWu"], st["dWd"], ws, need, stream)
            return
        wsf = st["ws_f"] if wl.backward else ws
        T.tsp_mlp_forward_ex(x, dev["A"], dev["Wu"], dev["B"], n, d, f, P, wl.act, dt, sched,
                             y, wsf, wsf.numel() if wl.backward else need, stream)
        if wl.backward:
            T.tsp_mlp_backward_ex(x, dev["A"], dev["Wu"], dev["B"], dev["dY"], n, d, f, P,
                                  wl.act, st["dX"], st["dWg"], st["dWu"], st["dWd"], ws, need,
                                  stream)

    config = {"workload": wl.name, "n_tokens": n, "d_model": d, "d_ff": f, "P": P,
              "act": wl.act, "schedule": sched,
              **({"backward": "saved activations" if saved_act else "recompute"}
                 if wl.backward else {}),
              "l2": "inputs larger than L2 (weights 3 x d x f bf16), no flush"
              if dt == "bf16" else "inputs fit in L2 (launch-latency bound), no flush"}
    return {"step": step, "inp": inp, "dev": dev, "Y": Y, "flops": workload_flops(wl),
            "dt": dt, "metric": metric_name(wl), "config": config,
            "kernel_flops": lambda k: kernel_flops_per_step(k, wl),
            "cpu_baseline": lambda: cpu_baseline(wl), "tokens": n}


def setup_attn(args, wl, T, stream):
    """The TSP attention block's forward through the C ABI."""
    inp = make_attn_inputs(wl)
    dev = {k: v.cuda() for k, v in inp.items()}
    n, d = wl.n, wl.d
    Y = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
    need = T.tsp_attn_workspace_size(n, d, wl.heads, wl.P)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def step(x=dev["X"], y=Y):
        T.tsp_attn_forward(x, dev["Wq"], dev["Wk"], dev["Wv"], dev["Wo"], n, d, wl.heads, wl.P,
                           wl.causal, y, ws, need, stream)

    fl = wl.flops()
    per_kernel = {"attn_core": fl["core"], "attn_core_causal": fl["core"],
                  "attn_proj": fl["projections"] * 3 / 4, "attn_out_proj": fl["projections"] / 4}
    config = {"workload": wl.name, "n_tokens": n, "d_model": d, "n_heads": wl.heads,
              "head_dim": wl.dh, "P": wl.P, "causal": wl.causal, "schedule": "tsp_attention",
              "l2": "inputs larger than L2 (X 268 MB, K/V of one head 16 MB), no flush"}
    return {"step": step, "inp": inp, "dev": dev, "Y": Y,
            "flops": fl["core"] + fl["projections"], "dt": "bf16",
            "metric": "TSP attention forward TFLOP/s", "config": config,
            "kernel_flops": lambda k: per_kernel[k],
            "cpu_baseline": lambda: attn_cpu_baseline(wl), "tokens": n}


def attn_oracle_sample(wl, inp, rows: int) -> dict:
    """The fp64 attention oracle, as it stands, on the first `rows` query rows
    of the block (every key and value of the sequence is projected for them),
    and the full step's CPU time extrapolated linearly in the number of query
    rows from two sample sizes."""
    from oracle import attention as OA
    args = [inp[k] for k in ("X", "Wq", "Wk", "Wv", "Wo")]
    times = {}
    for r in (max(1, rows // 4), rows):
        t0 = time.perf_counter()
        OA.attention_forward(*args, wl.heads, wl.causal, rows=list(range(r)))
        times[r] = time.perf_counter() - t0
    (r1, t1), (r2, t2) = sorted(times.items())
    per_row = max((t2 - t1) / max(r2 - r1, 1), 0.0)
    fixed = max(t1 - per_row * r1, 0.0)
    return {"rows_s": t2, "fixed_s": fixed, "per_row_s": per_row,
            "extrapolated_full_step_s": fixed + per_row * wl.n}


def attn_cpu_baseline(wl, rows=64):
    import oracle
    inp = make_attn_inputs(wl)
    parts = attn_oracle_sample(wl, inp, rows)
    full = parts["extrapolated_full_step_s"]
    fl = wl.flops()
    return {"value": (fl["core"] + fl["projections"]) / full / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows // 4} and {rows} query rows of {wl.name} (fp64 oracle: the "
                      f"keys and values of all {wl.n} tokens, then attention of those rows); "
                      f"full step extrapolated linearly in rows: {full:.1f} s",
            "extrapolated_full_step_s": full}


def attn_reference_arm(args, wl, rank):
    if rank != 0:
        return
    import oracle
    inp = make_attn_inputs(wl)
    rows = args.ref_rows or 64
    for _ in range(args.warmup):
        attn_oracle_sample(wl, inp, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        parts = attn_oracle_sample(wl, inp, rows)
    dt = (time.perf_counter() - t0) / args.steps
    fl = wl.flops()
    full = parts["extrapolated_full_step_s"]
    tflops = (fl["core"] + fl["projections"]) / full / 1e12
    line = {
        "impl": "reference", "metric": "TSP attention forward TFLOP/s", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded torch.randn)",
        "tokens_per_s": wl.n / full,
        "config": {"workload": wl.name, "n_tokens": wl.n, "d_model": wl.d, "n_heads": wl.heads,
                   "P": wl.P, "causal": wl.causal, "sample_rows": rows},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"first {rows // 4} and {rows} query rows per step",
                         "extrapolated_full_step_s": full},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=LLAMA8B.name,
                    choices=sorted(WORKLOADS) + sorted(ATTN_WORKLOADS))
    ap.add_argument("--sched", default=None,
                    choices=["weight_shards", "tsp_ring", "shard_passes", "fused", "tsp_ring_fused",
                             "shard_passes_fused"],
                    help="override the workload's schedule")
    ap.add_argument("--P", type=int, default=None,
                    help="override the workload's number of logical weight shards")
    ap.add_argument("--bwd-recompute", action="store_true",
                    help="fwd+bwd workloads: the inference forward and the backward that "
                         "recomputes the gate/up projection, instead of the training forward "
                         "that keeps its activations")
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="--impl reference: token rows (and, fwd+bwd, hidden columns) of the "
                         "oracle's sample per step (default 256, 64 for fwd+bwd and attention)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer loop (used for short profiler runs)")
    args = ap.parse_args()
    attn = args.workload in ATTN_WORKLOADS
    wl = ATTN_WORKLOADS[args.workload] if attn else WORKLOADS[args.workload]
    # traffic figures in the committed ncu summaries are for the workload's own P
    traffic_key = wl.name
    if args.P is not None and args.P != wl.P:
        wl = dataclasses.replace(wl, P=args.P)
        traffic_key = None

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        (attn_reference_arm if attn else reference_arm)(args, wl, rank)
        return

    import sequence_transformer_mlp_b200 as T

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    stream = torch.cuda.current_stream()
    run = (setup_attn if attn else setup_mlp)(args, wl, T, stream)
    step, inp, dev, Y, flops, dt = (run[k] for k in ("step", "inp", "dev", "Y", "flops", "dt"))

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK

    T.tsp_trace_reset()
    T.tsp_trace_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier()
    T.tsp_trace_enable(False)
    ms = e0.elapsed_time(e1) / args.steps
    kstats = T.tsp_trace_collect()
    T.tsp_trace_reset()
    status = T.tsp_poll_device_error()
    if status != T.TSP_OK:
        raise SystemExit(f"device error {T.STATUS_NAMES.get(status)} during the timed region")

    # end to end through the public call with host buffers: pinned X in, Y out
    if args.no_e2e:
        ms_e2e = float("nan")
        Xh = Yh = None
    else:
        ms_e2e, Xh, Yh = end_to_end(args, inp, dev, step, Y, stream, barrier)

    if dist is not None:
        ms, ms_e2e = max_over_ranks([ms, ms_e2e], dist, "cuda")

    clocks = clk.summary()
    timed_s = ms * args.steps * 1e-3
    clocks["timed_region_s"] = timed_s
    long_region = timed_s >= 1.0
    if rank == 0:
        pk = peaks()
        tflops = replica_throughput(world, flops, ms)
        # dominant kernel: the one with the largest share of traced time
        total_k = sum(v[1] for v in kstats.values())
        dom, (dom_launches, dom_ms) = max(kstats.items(), key=lambda kv: kv[1][1])
        launches_total = sum(v[0] for v in kstats.values())
        dom_flops_per_launch = run["kernel_flops"](dom) / (dom_launches / args.steps)
        achieved = dom_flops_per_launch / (dom_ms / dom_launches * 1e-3) / 1e12
        traffic = traffic_for(dom, traffic_key, dom_launches // args.steps) if traffic_key else None
        if dt == "f32":
            # fp32 FMA on the CUDA cores: peak = SMs x 128 lanes x 2 FLOP x max SM clock
            bound, peak, peak_src = "alu", fp32_alu_peak_tflops(clocks), "derived"
        else:
            bound, peak, peak_src = "tensor", pk["bf16_tflops"], pk["source"]
        line = {
            "metric": run["metric"],
            "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dt,
            "data": f"synthetic (seeded torch.randn, cast to {dt})",
            "tokens_per_s": world * run["tokens"] / (ms * 1e-3),
            "pct_of_bf16_peak": 100.0 * tflops / (world * pk["bf16_tflops"]),
            # a sustained (power-capped) peak applies only to a timed region of
            # seconds; a short burst is compared with the burst peak alone
            **({"pct_of_bf16_peak_sustained": 100.0 * tflops / (world * pk["bf16_tflops_sustained"])}
               if long_region else {}),
            "config": {**run["config"], "parallelism": f"replicas{world}"},
            "roofline": {"bound": bound, "kernel": dom, "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         **({"frac_of_sustained": achieved / pk["bf16_tflops_sustained"]}
                            if dt == "bf16" and long_region else {}),
                         "peak_source": peak_src, "traffic": traffic,
                         "flops_per_launch": dom_flops_per_launch,
                         "share_of_kernel_time": dom_ms / total_k if total_k else None},
            "kernels": {k: {"launches": v[0], "ms_per_launch": v[1] / v[0]}
                        for k, v in kstats.items()},
            "gpu_launches": launches_total,
            "e2e": None if Xh is None else {
                "value": replica_throughput(world, flops, ms_e2e), "unit": "TFLOP/s",
                "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
                "d2h_bytes_per_step": Yh.numel() * Yh.element_size(),
                "ms_per_step": ms_e2e},
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = run["cpu_baseline"]()
        print(json.dumps(line), flush=True)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def fp32_alu_peak_tflops(clocks: dict) -> float:
    """fp32 FMA peak of the device: SMs x 128 fp32 lanes x 2 FLOP x max SM clock."""
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    mhz = clocks.get("sm_max_mhz") or 1965.0
    return props.multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12


def kernel_flops_per_step(kernel: str, wl) -> float:
    """Algorithmic FLOPs one step spends in `kernel` (2 x rows x cols x K of each
    product it computes).  Per step the forward hidden kernel covers all n x f
    hidden units once and the down kernel all n x d outputs over K = d_ff,
    whatever the number of launches (chunks, ring steps) they are split into.
    The recompute backward's gate/up products are counted too: they run on the
    tensor cores like the rest (the fwd+bwd step's default path, the training
    forward that keeps its activations, has none)."""
    n, d, f = wl.n, wl.d, wl.f
    return {
        "fused_fwd_swiglu": 2 * 3 * n * d * f,
        "fused_fwd_gelu": 2 * 2 * n * d * f,
        "fwd_hidden_swiglu": 2 * 2 * n * d * f,
        "fwd_hidden_gelu": 2 * n * d * f,
        "fwd_hidden_swiglu_save": 2 * 2 * n * d * f,
        "fwd_hidden_gelu_save": 2 * n * d * f,
        "bwd_dh_factor_swiglu": 2 * n * d * f,
        "bwd_dh_factor_gelu": 2 * n * d * f,
        "down_accum_fwd": 2 * n * d * f,
        "fused_passes_swiglu": 2 * 3 * n * d * f,
        "fused_passes_gelu": 2 * 2 * n * d * f,
        "bwd_gate_up_swiglu": 2 * 2 * n * d * f,
        "bwd_gate_up_gelu": 2 * n * d * f,
        "bwd_dh_swiglu": 2 * n * d * f,
        "bwd_dh_gelu": 2 * n * d * f,
        "wgrad_down": 2 * n * d * f,
        "wgrad_gate_up": 2 * 2 * n * d * f,
        "wgrad_gelu_a": 2 * n * d * f,
        "dgrad_accum_swiglu": 2 * 2 * n * d * f,
        "dgrad_wgrad_swiglu": 2 * 2 * n * d * f + 2 * 2 * n * d * f,
        "dgrad_accum_gelu": 2 * n * d * f,
        "f32_hidden_swiglu": 2 * 2 * n * d * f,
        "f32_hidden_gelu": 2 * n * d * f,
        "f32_down": 2 * n * d * f,
    }[kernel]


if __name__ == "__main__":
    main()
