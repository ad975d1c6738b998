#!/usr/bin/env python
"""Benchmark: exact attention forward + backward, bf16, n = 16384 (B1 H16 D128).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the bf16 forward
(mea_attn_fwd) and the three backward phases (mea_attn_bwd_phase) on the
long-sequence workload B=1, H=16, N=16384, D=128, synthetic N(0,1) inputs.
The metric is TFLOP/s with the 4*B*H*N^2*D forward convention and 2.5x that
for the backward; `value` is the whole-job throughput over all ranks (each
rank runs its own independent batch: weak scaling, no data-path collective).

Rank 0 prints one JSON line.  Under torchrun (N > 1) ranks synchronise with a
barrier around the timed region and the slowest rank's device time is used.
`--impl reference` times the fp64 CPU oracle (the only reference there is) on
a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from synthetic_inputs import make_inputs, make_inputs_fp8, make_workload, custom  # noqa: E402

WORKLOAD = "long_16384_bf16"
METRIC = "attention fwd & fwd+bwd TFLOP/s, bf16 n=16384, % of B200 dense BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "exact_memory_efficient_b200", "csrc")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(names=None) -> str:
    """Hash of the CUDA sources (all of them, or the named files)."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")) and (names is None or name in names):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# the files whose text decides each timed kernel's device code: its own source
# and the device helpers it compiles (kernels.h holds host-side argument
# structs and the other kernels' declarations)
KERNEL_SOURCES = {
    "bwd_main_kernel": ("bwd_bf16.cu", "ptx.cuh"),
    "fwd_bf16_kernel": ("fwd_bf16.cu", "ptx.cuh"),
}


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's sources are unchanged since."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    base = kernel.split("<")[0]
    if not e or base not in KERNEL_SOURCES or e.get("src_sha") != source_sha(KERNEL_SOURCES[base]):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.fine = []
        self._stop = False
        self._thread = None
        self._nvml = None

    def _nvml_loop(self):
        # Finer record through NVML (read-only queries), every 5 ms: SM clock
        # and the event-reason mask (0x4 software power cap, 0x8 hardware
        # slowdown, 0x20 software thermal, 0x40 hardware thermal).
        import pynvml
        h = self._nvml
        while not self._stop:
            try:
                self.fine.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                  int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
            except Exception:  # noqa: BLE001
                return
            time.sleep(0.005)

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
        except Exception:  # noqa: BLE001 - NVML missing: keep the nvidia-smi record only
            return
        import threading
        self._thread = threading.Thread(target=self._nvml_loop, daemon=True)
        self._thread.start()

    def fine_summary(self):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=2)
        if not self.fine:
            return None
        sm = [c for c, _ in self.fine]
        return {"samples": len(sm), "period_ms": 5, "sm_mhz_median": statistics.median(sm), "sm_mhz_min": min(sm),
                "sw_power_cap_frac": round(sum(1 for _, r in self.fine if r & 0x4) / len(sm), 3),
                "hw_or_thermal_slowdown": any(r & (0x8 | 0x20 | 0x40) for _, r in self.fine)}

    def stop(self):
        fine = self.fine_summary()
        out = self._stop_smi()
        out["nvml_5ms"] = fine
        return out

    def _stop_smi(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [x for x in sm if x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


def cpu_oracle_sample(w, seed=0, q_rows=4096, min_seconds=0.0):
    """Time the fp64 oracle's forward + backward over q_rows query rows x all keys of one head,
    then of further heads until min_seconds of oracle time have passed (at most all heads)."""
    import oracle
    from synthetic_inputs import to_f64
    dt, heads = 0.0, 0
    while heads < w.B * w.H:
        q, k, v, do = make_inputs(custom(1, 1, q_rows, w.Nk, w.D, "bf16", True, name="oracle_sample"),
                                  seed * 1000 + heads)
        q2, k2, v2, do2 = (to_f64(x)[0, 0] for x in (q, k, v, do))
        t0 = time.perf_counter()
        oracle.attention_forward_2d(q2, k2, v2, w.scale)
        oracle.attention_backward_2d(q2, k2, v2, do2, w.scale)
        dt += time.perf_counter() - t0
        heads += 1
        if dt >= min_seconds:
            break
    flops = heads * 3.5 * 4.0 * q_rows * w.Nk * w.D
    cores = len(os.sched_getaffinity(0))
    return flops / dt / 1e12, dt, cores, (f"fp64 numpy oracle, forward then backward of {heads} of {w.B * w.H} "
                                          f"heads, {q_rows} of {w.Nq} query rows x all {w.Nk} keys each, D={w.D}")


def time_back_to_back(call, sets, stream, reps=30):
    """Device time of one call (microseconds): `reps` back-to-back calls over the input sets
    in turn, queued behind a sleep kernel so that the host has enqueued them all before the
    GPU reaches them, bracketed by one event pair on the launching stream."""
    for st in sets:
        call(st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(40_000_000)
    e0.record(stream)
    for r in range(reps):
        call(sets[r % len(sets)])
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps * 1e3


def naive_attention(q, k, v, scale):
    """The materialised-scores attention the method avoids: S = scale Q K^T, P = softmax(S),
    O = P V, as three plain PyTorch operations in the inputs' dtype (memory baseline only)."""
    s = torch.matmul(q, k.transpose(-1, -2)) * scale
    p = torch.softmax(s, dim=-1)
    return torch.matmul(p, v)


def measure_memory(m, w, dev, stream):
    """Peak device memory beyond inputs and outputs, measured by the caching allocator's peak
    (torch.cuda.max_memory_allocated) for four runs of the workload: the naive materialised
    attention forward, the same with an autograd backward, this library's forward (its extra
    is lse) and its forward + backward (lse + the backward workspace).  The library allocates
    nothing itself, which the driver's free-memory count around its calls confirms."""
    scale = w.scale
    q_h, k_h, v_h, do_h = make_inputs(w, 0)
    out = {}
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    def peak_above(base):
        torch.cuda.synchronize()
        return torch.cuda.max_memory_allocated(dev) - base

    # naive forward: the extra is everything beyond q, k, v and the output o
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    with torch.no_grad():
        o = naive_attention(q, k, v, scale)
    out["naive_fwd_peak_bytes"] = peak_above(base) - o.numel() * o.element_size()
    del o
    # naive forward + autograd backward: beyond q, k, v, dO, o and the three gradients
    qg, kg, vg = (x.clone().requires_grad_(True) for x in (q, k, v))
    do = do_h.to(dev)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    o = naive_attention(qg, kg, vg, scale)
    o.backward(do)
    grads = sum(x.grad.numel() * x.grad.element_size() for x in (qg, kg, vg))
    out["naive_fwdbwd_peak_bytes"] = peak_above(base) - o.numel() * o.element_size() - grads
    del o, qg, kg, vg
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    # this library: outputs allocated first, then the extra (lse, workspace) inside the window
    o = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    m.mea_attn_fwd(q, k, v, o, lse, scale, stream)
    out["ours_fwd_peak_bytes"] = peak_above(base)
    ws = torch.empty(m.mea_attn_bwd_workspace_size(w.B, w.H, w.Nq, w.Nk, w.D), dtype=torch.uint8, device=dev)
    m.mea_attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale, ws, stream)
    out["ours_fwdbwd_peak_bytes"] = peak_above(base)
    torch.cuda.synchronize()
    # device memory taken between the two snapshots by anything (the allocator's new
    # segments for lse and the workspace, and any allocation inside the library)
    out["ours_driver_free_delta_bytes"] = int(free0 - torch.cuda.mem_get_info(dev)[0])
    out["ours_allocator_extra_bytes"] = int(lse.numel() * 4 + ws.numel())
    out["naive_over_ours_fwd"] = round(out["naive_fwd_peak_bytes"] / out["ours_fwd_peak_bytes"], 1)
    out["naive_over_ours_fwdbwd"] = round(out["naive_fwdbwd_peak_bytes"] / out["ours_fwdbwd_peak_bytes"], 1)
    out["pages_tpu_ratios"] = {"inference": 59, "differentiation": 32, "n": 16384, "hardware": "TPUv3"}
    out["static_noalloc_scratch_bytes"] = int(m.MEA_NOALLOC_SCRATCH_BYTES)
    out["note"] = ("peaks from torch.cuda.max_memory_allocated above inputs and outputs; naive = bf16 "
                   "matmul -> softmax -> matmul (autograd for the backward); the static scratch of "
                   "mea_attn_bwd_noalloc is resident on every device that loads the library, whether "
                   "or not that entry point is called, and is listed apart")
    del q, k, v, do, o, dq, dk, dv, lse, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_workload(WORKLOAD)
    vals, times = [], []
    cores, sample = None, None
    for i in range(args.warmup + args.steps):
        v, dt, cores, sample = cpu_oracle_sample(w, seed=i % 3)
        if i >= args.warmup:
            vals.append(v)
            times.append(dt)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.median(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "N": w.Nq, "D": w.D, "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import exact_memory_efficient_b200 as m

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    m.load_library()
    peaks, peak_src = load_peaks()
    w = make_workload(args.workload)
    if w.dtype != "bf16" or not w.backward:
        raise SystemExit(f"--workload {args.workload}: the step needs a bf16 forward+backward workload")
    scale = w.scale

    # ---- inputs resident in HBM (one independent batch per rank)
    q_h, k_h, v_h, do_h = make_inputs(w, seed=rank)
    mem0 = torch.cuda.memory_allocated(dev)
    q, k, v, do = (x.to(dev) for x in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    mem_io = torch.cuda.memory_allocated(dev) - mem0
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(m.mea_attn_bwd_workspace_size(w.B, w.H, w.Nq, w.Nk, w.D), dtype=torch.uint8, device=dev)
    extra_bytes = lse.numel() * 4 + ws.numel()
    stream = torch.cuda.current_stream()

    def bwd(phase):
        m.mea_attn_bwd_phase(phase, q, k, v, o, lse, do, dq, dk, dv, scale, ws, stream)

    launches_per_step = 4  # fwd kernel + backward preprocess, main, finalise

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        m.mea_attn_fwd(q, k, v, o, lse, scale, stream)
        if ev is not None:
            ev[1].record(stream)
        bwd(m.MEA_BWD_PREPROCESS)
        if ev is not None:
            ev[2].record(stream)
        bwd(m.MEA_BWD_MAIN)
        if ev is not None:
            ev[3].record(stream)
        bwd(m.MEA_BWD_FINALIZE)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    st = m.mea_last_device_error(stream)
    if st != m.MEA_OK:
        raise RuntimeError(f"device error after warm-up: {m.mea_status_string(st)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    st = m.mea_last_device_error(stream)
    if st != m.MEA_OK:
        raise RuntimeError(f"device error in timed region: {m.mea_status_string(st)}")

    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    pre_ms = [e[1].elapsed_time(e[2]) for e in evs]
    main_ms = [e[2].elapsed_time(e[3]) for e in evs]
    fin_ms = [e[3].elapsed_time(e[4]) for e in evs]
    t = torch.tensor([total_ms, sum(fwd_ms), sum(main_ms)], dtype=torch.float64, device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, fwd_sum, main_sum = (float(x) for x in t.tolist())

    fwd_flops = w.fwd_flops()
    step_flops = 3.5 * fwd_flops
    value = world * args.steps * step_flops / (total_ms * 1e-3) / 1e12
    fwd_tf = fwd_flops / (statistics.mean(fwd_ms) * 1e-3) / 1e12
    bwd_ms = [a + b + c for a, b, c in zip(pre_ms, main_ms, fin_ms)]
    bwd_tf = 2.5 * fwd_flops / (statistics.mean(bwd_ms) * 1e-3) / 1e12
    main_avg_ms = statistics.mean(main_ms)
    main_tf = 2.5 * fwd_flops / (main_avg_ms * 1e-3) / 1e12

    # The dominant kernel is the backward main kernel; it runs inside a step
    # loop of total_ms; use the sustained GEMM peak once the loop is long.
    sustained = total_ms >= 1000.0
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    peak_step = peak

    # ---- end to end through the public API with host buffers (pinned).  Each
    # step copies q, k, v, dO in from pinned host memory and o, lse, dq, dk, dv
    # back out.  The heads are processed in chunks (a chunk is itself a
    # [B, H/c, N, D] call of the public API) so that the copies of one chunk
    # overlap the kernels of its neighbours: host-to-device on one stream,
    # kernels on two compute streams taken in turn (so one chunk's kernels can
    # fill the SMs left idle by its neighbour's last wave), device-to-host on a
    # fourth.
    e2e = None
    if not args.no_extras:
        pin = [x.pin_memory() for x in (q_h, k_h, v_h, do_h)]
        outs = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (q_h, k_h, v_h, q_h)]
        lse_h = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
        e2e_steps = max(1, min(args.steps, 20))
        n_chunks = 4 if (w.B == 1 and w.H % 4 == 0) else 1   # a head slice is contiguous when B = 1
        hc = w.H // n_chunks
        dbuf = [torch.empty_like(x, device=dev) for x in (q_h, k_h, v_h, do_h)]          # q, k, v, dO
        obuf = [torch.empty_like(x, device=dev) for x in (q_h, k_h, v_h, q_h)]          # o, dk, dv, dq
        lse_d = torch.empty(lse.shape, dtype=torch.float32, device=dev)
        ws_c = [torch.empty(m.mea_attn_bwd_workspace_size(w.B, hc, w.Nq, w.Nk, w.D), dtype=torch.uint8, device=dev)
                for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        s_cmp = [stream, torch.cuda.Stream(device=dev)]

        def heads(t, c):
            return t[:, c * hc:(c + 1) * hc]

        # per chunk: the last use of its input buffers by the kernels and the last
        # read of its output buffers by the copy-out (of the previous step), so
        # consecutive steps overlap without touching a buffer still in use
        used = [None] * n_chunks
        copied = [None] * n_chunks

        def e2e_step():
            for c in range(n_chunks):
                sc = s_cmp[c % 2]
                if used[c] is not None:
                    s_in.wait_event(used[c])
                with torch.cuda.stream(s_in):
                    for hsrc, ddst in zip(pin, dbuf):
                        heads(ddst, c).copy_(heads(hsrc, c), non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(s_in)
                sc.wait_event(ev_in)
                if copied[c] is not None:
                    sc.wait_event(copied[c])
                qd, kd, vd, dod = (heads(x, c) for x in dbuf)
                od, dkd, dvd, dqd = (heads(x, c) for x in obuf)
                ld = heads(lse_d, c)
                m.mea_attn_fwd(qd, kd, vd, od, ld, scale, sc)
                m.mea_attn_bwd(qd, kd, vd, od, ld, dod, dqd, dkd, dvd, scale, ws_c[c % 2], sc)
                used[c] = torch.cuda.Event()
                used[c].record(sc)
                s_out.wait_event(used[c])
                with torch.cuda.stream(s_out):
                    for dsrc, hdst in zip(obuf, outs):
                        heads(hdst, c).copy_(heads(dsrc, c), non_blocking=True)
                    heads(lse_h, c).copy_(ld, non_blocking=True)
                    copied[c] = torch.cuda.Event()
                    copied[c].record(s_out)

        e2e_step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_stream(stream)
        s_cmp[1].wait_stream(stream)
        for _ in range(e2e_steps):
            e2e_step()
        stream.wait_stream(s_cmp[1])
        stream.wait_stream(s_out)       # the timed region ends after the last copy-out
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
        st = m.mea_last_device_error(stream)
        if st != m.MEA_OK:
            raise RuntimeError(f"device error in the e2e steps: {m.mea_status_string(st)}")
        h2d = sum(x.numel() * x.element_size() for x in pin)
        d2h = sum(x.numel() * x.element_size() for x in outs) + lse_h.numel() * 4
        e2e = {"value": round(world * e2e_steps * step_flops / (float(e2e_ms.item()) * 1e-3) / 1e12, 3),
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": e2e_steps, "head_chunks": n_chunks,
               "note": "public API per head chunk; host-to-device, kernels (two streams, chunks in turn) and "
                       "device-to-host on separate streams; consecutive steps overlap"}

    # ---- fp32 SIMT rows (secondary measurements, single-query HBM roofline)
    rows = {}
    if rank == 0:
        rows[f"{w.name}_fwd"] = {"ms": round(statistics.mean(fwd_ms), 4), "TFLOP/s": round(fwd_tf, 1),
                                 "frac_of_peak": round(fwd_tf / peak, 3)}
        rows[f"{w.name}_bwd"] = {"ms": round(statistics.mean(bwd_ms), 4), "TFLOP/s": round(bwd_tf, 1),
                                 "frac_of_peak": round(bwd_tf / peak, 3),
                                 "phases_ms": {"preprocess": round(statistics.mean(pre_ms), 4),
                                               "main": round(main_avg_ms, 4),
                                               "finalize": round(statistics.mean(fin_ms), 4)}}
    if rank == 0 and not args.no_extras:
        # HBM-bound decode-shaped forwards.  Their K/V (67 MB) fit in L2, so each
        # is timed over three copies of its inputs (201 MB > L2) used in turn:
        # every launch reads K/V that the previous two launches evicted.  One
        # event pair brackets 30 back-to-back calls queued behind a sleep
        # kernel, so the time is the kernels' (plus the gaps between
        # consecutive launches), not the host's launch path.  The row's figure
        # is the split-KV entry (mea_attn_decode, caller workspace); the
        # workspace-free forward entry on the same inputs is reported beside it.
        for wname in ("single_query_f32", "decode_16384_bf16", "decode_gqa_32x8_16384_bf16"):
            wd = make_workload(wname)
            sets = []
            for copy in range(3):
                qd, kd, vd, _ = (x.to(dev) if x is not None else None for x in make_inputs(wd, copy))
                od, ld = m.attention_forward(qd, kd, vd, wd.scale)
                sets.append((qd, kd, vd, od, ld))
            ws_n = m.mea_attn_decode_workspace_size(wd.B, wd.H, wd.H_kv, wd.Nq, wd.Nk, wd.D, wd.torch_dtype)
            wsd = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)

            us = time_back_to_back(lambda s_: m.mea_attn_decode(*s_, wd.scale, wsd, stream), sets, stream)
            us_fwd = time_back_to_back(lambda s_: m.mea_attn_fwd_gqa(*s_, wd.scale, stream), sets, stream)
            byts = sum(x.numel() * x.element_size() for x in sets[0])
            rows[f"{wname}_fwd"] = {"us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
                                    "frac_of_hbm": round(byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3),
                                    "bytes": byts, "H_kv": wd.H_kv, "entry": "mea_attn_decode",
                                    "workspace_bytes": ws_n,
                                    "mea_attn_fwd_gqa_us": round(us_fwd, 2),
                                    "note": "30 back-to-back calls over 3 input copies (201 MB > L2)"}
            del sets
        # grouped-query forward + backward (32 query heads over 8 key/value heads)
        wg = make_workload("gqa_32x8_4096_bf16")
        qg, kg, vg, dog = (x.to(dev) for x in make_inputs(wg, 0))
        og, lg = m.attention_forward(qg, kg, vg, wg.scale)
        wsg = torch.empty(m.mea_attn_bwd_gqa_workspace_size(wg.B, wg.H, wg.H_kv, wg.Nq, wg.Nk, wg.D),
                          dtype=torch.uint8, device=dev)
        grads = [torch.empty_like(x) for x in (qg, kg, vg)]
        for _ in range(3):
            m.mea_attn_fwd_gqa(qg, kg, vg, og, lg, wg.scale)
            m.mea_attn_bwd_gqa(qg, kg, vg, og, lg, dog, *grads, wg.scale, wsg)
        reps = 10
        ev_g = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        for e in ev_g:
            e[0].record(stream)
            m.mea_attn_fwd_gqa(qg, kg, vg, og, lg, wg.scale)
            e[1].record(stream)
            m.mea_attn_bwd_gqa(qg, kg, vg, og, lg, dog, *grads, wg.scale, wsg)
            e[2].record(stream)
        torch.cuda.synchronize()
        f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_g)
        b_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev_g)
        rows[f"{wg.name}_fwd"] = {"ms": round(f_ms, 4), "TFLOP/s": round(wg.fwd_flops() / (f_ms * 1e-3) / 1e12, 1),
                                  "frac_of_peak": round(wg.fwd_flops() / (f_ms * 1e-3) / 1e12 / peak, 3)}
        rows[f"{wg.name}_bwd"] = {"ms": round(b_ms, 4), "TFLOP/s": round(wg.bwd_flops() / (b_ms * 1e-3) / 1e12, 1),
                                  "frac_of_peak": round(wg.bwd_flops() / (b_ms * 1e-3) / 1e12 / peak, 3),
                                  "note": f"mean of {reps}; inputs ({wg.H}+2x{wg.H_kv} heads) fit in L2"}
        del qg, kg, vg, dog, og, lg, wsg, grads
        # the head-dim-64 configurations (B4 H8 N4096 and B32 H8 N512), forward and
        # backward through the public API, timed on the device like the decode rows:
        # three copies of the inputs (3 x 67 MB > L2) used in turn, 30 back-to-back
        # calls queued behind a sleep kernel and bracketed by one event pair.  Their
        # roofline is max(compute at the measured bf16 peak, compulsory bytes at the
        # measured HBM copy rate): the encoder-shaped batch sits near the ridge.
        for wname in ("mha_4k_bf16", "encoder_512_bf16"):
            wx = make_workload(wname)
            sets = []
            for copy in range(3):
                qx, kx, vx, dox = (x.to(dev) for x in make_inputs(wx, copy))
                ox, lx = m.attention_forward(qx, kx, vx, wx.scale)
                sets.append((qx, kx, vx, dox, ox, lx, [torch.empty_like(x) for x in (qx, kx, vx)]))
            wsx = torch.empty(m.mea_attn_bwd_workspace_size(wx.B, wx.H, wx.Nq, wx.Nk, wx.D), dtype=torch.uint8,
                              device=dev)
            f_us = time_back_to_back(lambda s_: m.mea_attn_fwd(s_[0], s_[1], s_[2], s_[4], s_[5], wx.scale, stream),
                                     sets, stream)
            b_us = time_back_to_back(lambda s_: m.mea_attn_bwd(s_[0], s_[1], s_[2], s_[4], s_[5], s_[3], *s_[6],
                                                               wx.scale, wsx, stream), sets, stream)
            elt = 2  # bf16
            tensor_bytes = wx.B * wx.H * wx.Nq * wx.D * elt
            rows_bytes = wx.B * wx.H * wx.Nq * 4
            fwd_bytes = 4 * tensor_bytes + rows_bytes            # q, k, v read; o written; lse written
            bwd_bytes = 8 * tensor_bytes + 2 * rows_bytes        # q, k, v, o, dO read; dq, dk, dv written; lse, D
            for kind, us, flops, byts in (("fwd", f_us, wx.fwd_flops(), fwd_bytes),
                                          ("bwd", b_us, wx.bwd_flops(), bwd_bytes)):
                t_tensor = flops / (peak * 1e12) * 1e6
                t_hbm = byts / (peaks["hbm_gbs"] * 1e9) * 1e6
                rows[f"{wname}_{kind}"] = {
                    "us": round(us, 2), "TFLOP/s": round(flops / (us * 1e-6) / 1e12, 1),
                    "frac_of_peak": round(flops / (us * 1e-6) / 1e12 / peak, 3),
                    "roofline_us": round(max(t_tensor, t_hbm), 2), "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                    "frac_of_roofline": round(max(t_tensor, t_hbm) / us, 3), "compulsory_bytes": byts,
                    "note": f"D={wx.D}; 30 back-to-back calls over 3 input copies (> L2) behind a sleep kernel"}
            del sets, wsx
        # merge of a 4-way key split of the step's workload (HBM-bound): reads four
        # [B,H,N,D] bf16 parts and their lse, writes the merged o and lse
        R = 4
        parts_o = [torch.randn(w.B, w.H, w.Nq, w.D, device=dev).to(torch.bfloat16) for _ in range(R)]
        parts_l = [torch.randn(w.B, w.H, w.Nq, device=dev) for _ in range(R)]
        oc = torch.empty_like(parts_o[0])
        lc = torch.empty_like(parts_l[0])
        for _ in range(3):
            m.mea_attn_combine(parts_o, parts_l, oc, lc)
        reps = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            m.mea_attn_combine(parts_o, parts_l, oc, lc)
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / reps * 1e3
        byts = (R + 1) * (parts_o[0].numel() * 2 + parts_l[0].numel() * 4)
        rows[f"combine_{R}way_{w.name}"] = {"us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
                                             "frac_of_hbm": round(byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3),
                                             "bytes": byts, "note": "20 back-to-back launches; 272 MB of parts > L2"}
        del parts_o, parts_l, oc, lc
        # FP8 forward (e4m3 Q, K; bf16 V, O) on the step's workload
        q8, k8, v8, qd8, kd8 = make_inputs_fp8(w, 0)
        q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
        o8 = torch.empty((w.B, w.H, w.Nq, w.D), dtype=torch.bfloat16, device=dev)
        l8 = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        for _ in range(3):
            m.mea_attn_fwd_fp8(q8, k8, v8, o8, l8, scale, qd8, kd8)
        reps = 10
        ev8 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in ev8:
            e0.record(stream)
            m.mea_attn_fwd_fp8(q8, k8, v8, o8, l8, scale, qd8, kd8)
            e1.record(stream)
        torch.cuda.synchronize()
        f8_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev8)
        f8_tf = w.fwd_flops() / (f8_ms * 1e-3) / 1e12
        # half the flops (S = Q K^T) at the e4m3 rate (2x bf16, the nominal ratio), half at bf16
        mixed_peak = peak / 0.75
        rows[f"{w.name}_fp8_fwd"] = {"ms": round(f8_ms, 4), "TFLOP/s": round(f8_tf, 1),
                                     "frac_of_peak": round(f8_tf / mixed_peak, 3),
                                     "peak": round(mixed_peak, 1),
                                     "note": "e4m3 Q, K; bf16 V, O; 4*B*H*N^2*D flops; peak = measured bf16 "
                                             "burst / 0.75 (S at 2x the bf16 rate, P V at bf16)"}
        del q8, k8, v8, o8, l8

    # ---- extra memory versus a materialised-scores attention (measured peaks)
    memory = {"extra_bytes_ours": extra_bytes, "io_bytes": mem_io,
              "naive_score_matrix_fp32_bytes": w.B * w.H * w.Nq * w.Nk * 4,
              "static_noalloc_scratch_bytes": int(m.MEA_NOALLOC_SCRATCH_BYTES)}
    if rank == 0 and not args.no_extras:
        del q, k, v, do, o, dq, dk, dv, lse, ws
        memory.update(measure_memory(m, w, dev, stream))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.no_extras:
        cv, cdt, cores, sample = cpu_oracle_sample(w, min_seconds=10.0)
        cpu = {"value": round(cv, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(cdt, 2)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.Nq, "D": w.D, "scale": scale,
                       "global_batch": world * w.B, "seq_len": w.Nq, "parallelism": f"replicas x{world}",
                       "step": "mea_attn_fwd + mea_attn_bwd (3 phases)",
                       "l2": "inputs larger than L2 (q, k, v, o, dO, dq, dk, dv + fp32 dQ workspace), no flush"},
            "pct_of_peak": round(100 * value / world / peak_step, 2),
            "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": round(bwd_tf, 2),
            "roofline": {"kernel": f"bwd_main_kernel<{w.D}>", "bound": "tensor", "achieved": round(main_tf, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(main_tf / peak, 4),
                         "traffic": ncu_traffic(f"bwd_main_kernel<{w.D}>"),
                         "peak_source": f"{peak_src} {'bf16_tflops_sustained' if sustained else 'bf16_tflops'}",
                         "flops_per_launch": 2.5 * fwd_flops},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clk, "memory": memory, "rows": rows, "src_sha": source_sha(),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_profile(name: str) -> int:
    """Three forward (+ backward) calls of one workload through the public API, untimed.
    Forward-only workloads go through mea_attn_decode, the entry the decode rows time
    (it is the plain forward when a head has more than 8 query rows)."""
    import exact_memory_efficient_b200 as m
    w = make_workload(name)
    torch.cuda.set_device(0)
    q, k, v, do = (x.cuda() if x is not None else None for x in make_inputs(w, 0))
    for _ in range(3):
        if do is None:
            m.attention_decode(q, k, v, w.scale)
            continue
        o, lse = m.attention_forward(q, k, v, w.scale)
        m.attention_backward(q, k, v, o, lse, do, w.scale)
    st = m.mea_last_device_error()
    if st != m.MEA_OK:
        raise RuntimeError(m.mea_status_string(st))
    print(f"profile {name}: ok")
    return 0


def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload name from synthetic_inputs.WORKLOADS (bf16 with backward); the default is the "
                         "headline workload, others are for profiling captures")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the end-to-end, fp32-row and CPU-baseline measurements (profiling captures)")
    ap.add_argument("--profile", metavar="WORKLOAD", default=None,
                    help="no timing: run this workload's forward (and backward, if it has one) three times and "
                         "exit; the command profiling captures wrap (forward-only workloads: mea_attn_decode)")
    return ap


def main():
    ap = build_parser()
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile is not None:
        return run_profile(args.profile)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
