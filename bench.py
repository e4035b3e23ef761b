"""Benchmark of bf16 shifted local window attention on B200.

Prints one JSON line.  A step is one call of the library's window attention on
one batch of the workload (for workloads with global memory: pooling + window
attention); inputs are seeded and synthetic.

Kernel time: every step is bracketed by CUDA events on the launching stream.
Before each step the L2 is evicted (a 256 MiB write, then a 256 MiB read of
another buffer, so no dirty lines are left to be written back during the
timed kernel) and a short device sleep
is queued, so the event pair measures the kernel and not the host-side launch
preparation; neither the flush nor the sleep is inside the events.  Reported:
algorithmic TFLOP/s (4*B*H*N*(m+P)*d flops per step), latency, the dominant
kernel's roofline fraction, and the realised full-attention / window-attention
speedup against the theoretical N/m (N/(m+P) with global memory).

e2e: the same metric through the public API with host buffers: every step
copies its pinned q, k, v (and text tokens) to the device, makes the call, and
copies its output back, all inside the timed region.  Steps are pipelined over
two device buffer sets on three streams (copy in, compute, copy out), as a
serving loop would run them: step i + 1's inputs travel while step i computes
and its output travels back (PCIe is full duplex).

cpu_baseline / --impl reference: the CPU fp64 oracle timed on the host cores on
a bounded sample of the same workload (all queries of a few heads).

Multi-GPU (torchrun): each rank runs an independent replica of the workload
(the path has no exchange step); the time is the max over ranks.

--backward: the same timing for the gradients (dq, dk, dv) of the workload's
window attention (with its pooled memory, if any) for a random output gradient.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from basa_synth import WORKLOADS, text_inputs, workload_inputs  # noqa: E402

METRIC = "window-attn latency (ms) & TFLOPS/% bf16 peak; realised/theoretical N/m speedup"
DEFAULT_WORKLOAD = "flux2048"
_CSRC = os.path.join(ROOT, "sparse_attention_diffusion_basa_b200", "csrc")
# the source files whose device code each profiled kernel is built from
KERNEL_SOURCES = {
    "tc_attn_kernel": [os.path.join(_CSRC, "basa_tc.cu"), os.path.join(_CSRC, "tc_device.cuh")],
    "pool_kernel": [os.path.join(_CSRC, "basa_pool.cu")],
    "tc_bwd_kernel": [os.path.join(_CSRC, "basa_tc_bwd.cu"), os.path.join(_CSRC, "tc_device.cuh")],
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _source_hash(paths):
    h = hashlib.sha256()
    for path in paths:
        h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def _traffic(kernel_key, workload):
    """Per-launch DRAM bytes from a committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        t = json.load(open(path))
        e = t[kernel_key][workload]
        if e["source_sha"] != _source_hash(KERNEL_SOURCES[kernel_key]):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def sdpa_window_attn(q, k, v, window, shift):
    """Context comparator (not the library): the backend-agnostic route the
    BASA page describes, i.e. roll the grid by -shift, reshape it into windows,
    run torch's scaled_dot_product_attention (its own kernel choice) on every
    window, reshape back and roll by +shift.  q, k, v: [B, T, Hg, Wg, H, d]."""
    import torch.nn.functional as F
    B, T, Hg, Wg, H, d = q.shape
    wt, wh, ww = window
    nt, nh, nw = T // wt, Hg // wh, Wg // ww
    dims = (1, 2, 3)

    def to_windows(x):
        x = torch.roll(x, tuple(-s for s in shift), dims)
        x = x.view(B, nt, wt, nh, wh, nw, ww, H, d).permute(0, 1, 3, 5, 7, 2, 4, 6, 8)
        return x.reshape(B * nt * nh * nw, H, wt * wh * ww, d)

    o = F.scaled_dot_product_attention(to_windows(q), to_windows(k), to_windows(v))
    o = o.view(B, nt, nh, nw, H, wt, wh, ww, d).permute(0, 1, 5, 2, 6, 3, 7, 4, 8)
    return torch.roll(o.reshape(B, T, Hg, Wg, H, d), tuple(shift), dims)


def sdpa_full_attn(q, k, v):
    """Context comparator: torch's scaled_dot_product_attention over all tokens."""
    import torch.nn.functional as F
    B, T, Hg, Wg, H, d = q.shape
    f = lambda x: x.reshape(B, T * Hg * Wg, H, d).transpose(1, 2)
    return F.scaled_dot_product_attention(f(q), f(k), f(v)).transpose(1, 2)


def sdpa_comparators(q, k, v, w, shift, steps, flush, world):
    """Times the two SDPA routes under the first torch attention backend that
    runs them (cuDNN, flash, memory-efficient, then the unfused math path)."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION,
                    SDPBackend.EFFICIENT_ATTENTION, SDPBackend.MATH):
        try:
            with sdpa_kernel(backend):
                sdpa_window_attn(q, k, v, w.window, shift)
                sdpa_full_attn(q, k, v)
                torch.cuda.synchronize()
                t_sw = time_steps(lambda: sdpa_window_attn(q, k, v, w.window, shift), steps, flush)
                t_sf = time_steps(lambda: sdpa_full_attn(q, k, v), steps, flush)
        except RuntimeError:
            continue
        return {"torch_sdpa_window_roll_reshape_ms": max_over_ranks(sum(t_sw) / len(t_sw), world),
                "torch_sdpa_full_ms": max_over_ranks(sum(t_sf) / len(t_sf), world),
                "backend": backend.name,
                "note": "torch.nn.functional.scaled_dot_product_attention; context only, not "
                        "part of the library"}
    return None


def workload_numbers(w, shift):
    """Algorithmic flops and bytes of one step, and the full-attention cost ratio.

    Image queries see m window keys + P pooled + L text keys; text queries see all
    N + L tokens.  Bytes: q, k, v read and out written once, image and text."""
    B, T, Hg, Wg, H, d = w.shape()
    N, m, P, L = w.N, w.m, w.P, w.text
    pairs = N * (m + P + L) + L * (N + L)
    flops = 4.0 * B * H * d * pairs
    esize = {"bf16": 2, "e4m3": 1}.get(w.dtype, 4)  # q, k, v elements
    osize = 2 if w.dtype == "e4m3" else esize        # the output (bf16 for e4m3 inputs)
    bytes_ = B * H * (N + L) * d * (3.0 * esize + osize)
    theo = (N + L) ** 2 / pairs  # full attention over all tokens / this step
    return flops, bytes_, N, m, P, theo


class ClockSampler:
    """SM clock and throttle-reason sampling (NVML, every ~2 ms) during the timed region."""

    REASONS = {  # NVML clocks-event-reason bits
        0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap",
    }

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self._stop = None
        self._thread = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            # NVML numbers devices as the driver does; honour CUDA_VISIBLE_DEVICES
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.dev]) if vis else self.dev
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return None
        mhz = [m for m, _ in self.samples]
        reasons = sorted({name for _, rs in self.samples for bit, name in self.REASONS.items()
                          if rs & bit})
        return {"sm_mhz": float(np.median(mhz)), "sm_min_mhz": float(min(mhz)),
                "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                "samples": len(self.samples), "source": "nvml"}


def _sleep_cycles(us):
    # torch.cuda._sleep spins for a number of cycles; ~2 GHz upper bound on the clock
    torch.cuda._sleep(int(us * 2000))


class L2Flush:
    """Evicts the L2 (126 MB on B200) between timed steps.

    A 256 MiB write replaces every line, then a 256 MiB read of another buffer
    replaces the dirty lines the write left, so the timed kernel starts with an
    L2 that holds none of its data and owes no write-backs of someone else's.
    Both run outside the timing events.
    """

    def __init__(self, device, nbytes=256 << 20):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.r = torch.zeros(nbytes // 4, dtype=torch.int32, device=device)
        self.i = 0

    def __call__(self):
        self.i += 1
        self.w.fill_(self.i & 0xFF)
        self.sink = torch.amax(self.r)


def time_steps(fn, steps, flush, sleep_us=200.0):
    """Per-step device time (ms) of fn() with an L2 flush and a sleep before each step."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush()
        if sleep_us > 0:
            _sleep_cycles(sleep_us)
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _head(x, h):
    """Batch 0, head h of an image [B, T, Hg, Wg, H, d] or text [B, L, H, d] tensor."""
    return np.ascontiguousarray(x[:1, ..., h:h + 1, :])


def run_oracle_sample(w, shift, q, k, v, heads, threads=0):
    """Oracle on all queries of `heads` heads (batch 0); returns (seconds, flops).
    Joint workloads: every image and text query of each sampled head."""
    import oracle
    B, T, Hg, Wg, H, d = w.shape()
    N = w.N
    if w.text:
        L = w.text
        qt, kt, vt = (oracle.as_f64(x) for x in text_inputs(w, len(w.shifts) - 1))
        qf, kf, vf = oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v)
        prm = oracle.OracleParams(1, T, Hg, Wg, 1, d, w.window, shift)
        dt = 0.0
        for h in heads:
            args = [_head(x, h) for x in (qf, kf, vf, qt, kt, vt)]
            t0 = time.perf_counter()
            oracle.joint_attn(*args, prm, threads=threads)
            dt += time.perf_counter() - t0
        return dt, 4.0 * len(heads) * (N * (w.m + L) + L * (N + L)) * d
    sel = np.array([[0, n, h] for h in heads for n in range(N)], dtype=np.int64)
    prm = oracle.OracleParams(B, T, Hg, Wg, H, d, w.window, shift, w.pool)
    qf, kf, vf = oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v)
    kp = vp = None
    if w.P:
        kp = oracle.pool_kv(kf, prm)
        vp = oracle.pool_kv(vf, prm)
    t0 = time.perf_counter()
    oracle.window_attn(qf, kf, vf, prm, kp=kp, vp=vp, select=sel, threads=threads)
    dt = time.perf_counter() - t0
    return dt, 4.0 * len(sel) * (w.m + w.P) * d


def run_oracle_bwd_sample(w, shift, q, k, v, h):
    """The oracle's backward (gradients of every input) for batch 0, head h;
    returns (seconds, flops).  Joint workloads: image and text gradients."""
    import oracle
    B, T, Hg, Wg, H, d = w.shape()
    N, L = w.N, w.text
    rng = np.random.Generator(np.random.PCG64(7))
    qf, kf, vf = (_head(oracle.as_f64(x), h) for x in (q, k, v))
    g = rng.standard_normal(qf.shape)
    prm = oracle.OracleParams(1, T, Hg, Wg, 1, d, w.window, shift, w.pool)
    t0 = time.perf_counter()
    if L:
        qt, kt, vt = (_head(oracle.as_f64(x), h) for x in text_inputs(w, len(w.shifts) - 1))
        gt = rng.standard_normal(qt.shape)
        t0 = time.perf_counter()
        oracle.joint_attn_bwd(qf, kf, vf, qt, kt, vt, g, gt, prm)
    else:
        oracle.window_attn_bwd(qf, kf, vf, g, prm)
    dt = time.perf_counter() - t0
    return dt, 10.0 * (N * (w.m + w.P + L) + L * (N + L)) * d


def cpu_baseline(w, shift, q, k, v, budget_s=12.0):
    import oracle
    oracle.build_oracle()
    cores = oracle.max_threads()
    dt1, fl1 = run_oracle_sample(w, shift, q, k, v, [0])
    nheads = max(1, min(w.H, int(budget_s / max(dt1, 1e-3))))
    heads = list(range(nheads))
    dt, fl = run_oracle_sample(w, shift, q, k, v, heads)
    reps = 1
    # a whole batch finishing well inside the budget: repeat it for a steadier number
    while nheads == w.H and dt < budget_s * 0.75 and reps < 16:
        dti, fli = run_oracle_sample(w, shift, q, k, v, heads)
        dt, fl, reps = dt + dti, fl + fli, reps + 1
    res = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
           "sample": f"all {w.N} queries of {nheads} of {w.H} heads, batch 0, shift {shift}"
                     + (f", with the {w.text} text queries of those heads" if w.text else "")
                     + f", {reps} run(s); {dt:.2f} s fp64 on {cores} host threads"}
    # the same oracle on one host thread, on one head, where that takes a few
    # seconds at most (the small and the FLUX image workloads)
    if fl1 <= 3e9:
        dt1t, fl1t = run_oracle_sample(w, shift, q, k, v, [0], threads=1)
        res["one_thread"] = {"value": fl1t / dt1t / 1e12, "unit": "TFLOP/s", "cores": 1,
                             "sample": f"all {w.N} queries of head 0, batch 0; {dt1t:.2f} s fp64"
                                       " on 1 host thread"}
    return res


def main_backward(args, world, rank, local):
    """Backward of the workload's window attention: dq, dk, dv for a random dout
    (joint workloads: also dqt, dkt, dvt for a random dout_t)."""
    import sparse_attention_diffusion_basa_b200 as basa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    shift = w.shifts[-1]
    q, k, v = workload_inputs(w, len(w.shifts) - 1)
    dq, dk, dv = (x.to(dev) for x in (q, k, v))
    g = torch.randn(dq.shape, generator=torch.Generator().manual_seed(7)).to(dq.dtype).to(dev)
    flush = L2Flush(dev)
    L = w.text
    if L:
        qt, kt, vt = (x.to(dev) for x in text_inputs(w, len(w.shifts) - 1))
        gt = torch.randn(qt.shape, generator=torch.Generator().manual_seed(8)).to(qt.dtype).to(dev)
        out, out_t, lse, lse_t = basa.joint_attn(dq, dk, dv, qt, kt, vt, w.window, shift,
                                                 return_lse=True)
        need = basa.joint_bwd_workspace_size(w.shape(), dq.dtype, w.window, shift, L)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        step = lambda: basa.joint_attn_bwd(dq, dk, dv, qt, kt, vt, out, out_t, g, gt, lse, lse_t,
                                           w.window, shift, workspace=ws)
    else:
        out, lse = basa.window_attn(dq, dk, dv, w.window, shift, w.pool, return_lse=True)
        ws = torch.empty(max(basa.bwd_workspace_size(w.shape(), dq.dtype, w.window, shift,
                                                     w.pool), 1), dtype=torch.uint8, device=dev)
        step = lambda: basa.window_attn_bwd(dq, dk, dv, out, g, lse, w.window, shift, w.pool,
                                            workspace=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    clocks.start()
    t = time_steps(step, args.steps, flush)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    assert basa.get_status() == 0
    ms = max_over_ranks(sum(t) / len(t), world)
    B, T, Hg, Wg, H, d = w.shape()
    Hkv = H
    # five contractions per query and key: S (recomputed), dP, dV, dQ, dK (the
    # forward has two); keys = the window's m plus the P pooled tokens (joint:
    # image queries see m + L keys, text queries N + L)
    flops = 10.0 * B * H * (w.N * (w.m + w.P + L) + L * (w.N + L)) * d
    # q, k, v, out, dout read once; dq, dk, dv written once; per query row the
    # lse read and D = rowsum(dout * out) written and read once (12 B); with
    # pooled memory the pooled K, V (bf16) and their fp32 gradients written and
    # read once; text tokens count as image tokens do
    nbytes = 2.0 * B * (w.N + L) * d * ((3 * H + 2 * Hkv) + (H + 2 * Hkv)) \
        + 12.0 * B * H * (w.N + L) + 2.0 * B * w.P * Hkv * d * (2 * 2 + 2 * 4)
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = _peaks()
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"]}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof.update({"peak_source": peaks["source"] + " (MEASURED_PEAKS.json, burst)",
                 "traffic": None, "roofline_ms": 1e3 * max(t_tensor, t_hbm),
                 "kernel": ("whole joint backward: bwd_prep (image, text rows), tc_bwd_kernel "
                            "(text keys' dK, dV; image dQ; text dQ; window dK, dV), "
                            "text_grad_round_kernel") if L else
                           ("whole backward: bwd_prep, tc_bwd_kernel (dQ), tc_bwd_kernel (dK, dV)"
                            + (", pool_kernel, tc_bwd_kernel (pooled dK, dV)" if w.P else ""))})
    line = {"metric": "window-attn backward latency (ms) & TFLOP/s", "value": world * tflops,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 (tensor cores, fp32 accumulate)" if w.dtype == "bf16" else w.dtype,
            "data": "synthetic",
            "config": {"workload": f"{w.name} backward", "N": w.N, "m": w.m, "P": w.P, "L": L,
                       "l2": "evicted before every step (256 MiB write, then 256 MiB read; outside the events)"},
            "roofline": roof,
            "gpu_launches": (7 if L else 5 if w.P else 3) * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        torch.distributed.destroy_process_group()
    return 0


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() and args.impl != "reference" else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def arm_config(w, shift, world):
    """The workload description both arms print in their JSON line."""
    _, _, N, m, P, _ = workload_numbers(w, shift)
    L = w.text
    return {"workload": f"{w.name}: B={w.B} grid {w.T}x{w.Hg}x{w.Wg} H={w.H} d={w.d} "
                        f"window {'x'.join(map(str, w.window))} shift {shift} "
                        f"pool {w.pool}" + (f" text {L}" if L else ""),
            "N": N, "m": m, "P": P, "global_batch": w.B * world,
            "l2": "evicted before every step (256 MiB write, then 256 MiB read; outside the events)",
            "parallelism": f"replicas x{world}"}


def main_reference(args, world, rank):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    oracle.build_oracle()
    w = WORKLOADS[args.workload]
    shift = w.shifts[-1]
    q, k, v = workload_inputs(w, len(w.shifts) - 1)
    cores = oracle.max_threads()
    flops_step = 0.0
    if args.backward:  # the backward arm: the oracle's gradients, single-threaded C
        sample = lambda: run_oracle_bwd_sample(w, shift, q, k, v, 0)
        metric, cores = "window-attn backward latency (ms) & TFLOP/s", 1
        what = (f"gradients of every input, head 0 of {w.H}, batch 0, per step"
                + (f" (with its {w.text} text tokens)" if w.text else ""))
    else:
        sample = lambda: run_oracle_sample(w, shift, q, k, v, [0])
        metric = METRIC
        what = (f"all {w.N} queries of head 0 of {w.H}, batch 0, per step"
                + (f", and its {w.text} text queries" if w.text else ""))
    for _ in range(args.warmup):
        sample()
    times = []
    for _ in range(args.steps):
        dt, fl = sample()
        times.append(dt)
        flops_step = fl
    total = sum(times)
    val = flops_step * args.steps / total / 1e12
    line = {"impl": "reference", "metric": metric, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(w, shift, world),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": what},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="basa", choices=["basa", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--full-steps", type=int, default=5)
    ap.add_argument("--no-comparators", action="store_true",
                    help="skip the torch SDPA context timings")
    ap.add_argument("--no-blocks", action="store_true",
                    help="skip the per-block timings of a multi-block shift schedule")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward (dq, dk, dv) of the workload's window attention")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = main_reference(args, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc

    if args.backward:
        return main_backward(args, world, rank, local)

    import sparse_attention_diffusion_basa_b200 as basa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    blocks = list(range(len(w.shifts)))
    # the timed step uses the workload's last shift (the wrapped case where shifts differ)
    blk = blocks[-1]
    shift = w.shifts[blk]
    q, k, v = workload_inputs(w, blk)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    dq, dk, dv = (x.to(dev) for x in (q, k, v))
    odt = torch.bfloat16 if dq.dtype == torch.float8_e4m3fn else dq.dtype  # e4m3 -> bf16 out
    out = torch.empty(dq.shape, dtype=odt, device=dev)
    outh = torch.empty(qh.shape, dtype=odt).pin_memory()
    ws_bytes = basa.workspace_size(w.shape(), dq.dtype, w.window, shift, w.pool)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    flops, bytes_, N, m, P, theo = workload_numbers(w, shift)
    L = w.text

    def call(ins, outs):
        basa.window_attn(*ins, w.window, shift, w.pool, out=outs[0],
                         workspace=ws if ws_bytes else None)

    def step():
        call((dq, dk, dv), (out,))

    def step_full():
        basa.full_attn(dq, dk, dv, out=out)

    host_in, host_out = [(qh, dq), (kh, dk), (vh, dv)], [(outh, out)]
    if L:  # joint text + image block
        qt, kt, vt = text_inputs(w, blk)
        dqt, dkt, dvt = (x.to(dev) for x in (qt, kt, vt))
        out_t = torch.empty_like(dqt)
        host_in += [(x.pin_memory(), y) for x, y in ((qt, dqt), (kt, dkt), (vt, dvt))]
        host_out.append((torch.empty_like(qt).pin_memory(), out_t))
        # full attention over every image and text token, as one flat grid
        cat = [torch.cat([a.reshape(w.B, N, w.H, w.d), b], 1).reshape(w.B, 1, 1, N + L, w.H, w.d)
               for a, b in ((dq, dqt), (dk, dkt), (dv, dvt))]
        out_cat = torch.empty_like(cat[0])
        # the text pass's split workspace, allocated once outside the timed steps
        jws = torch.empty(max(basa.joint_workspace_size(w.shape(), dq.dtype, w.window, shift, L), 1),
                          dtype=torch.uint8, device=dev)

        def call(ins, outs):
            basa.joint_attn(*ins, w.window, shift, out=outs[0], out_t=outs[1], workspace=jws)

        def step():
            call((dq, dk, dv, dqt, dkt, dvt), (out, out_t))

        def step_full():
            basa.full_attn(*cat, out=out_cat)

    # two device buffer sets for the pipelined end-to-end steps
    sets = [([d_ for _, d_ in host_in], [d_ for _, d_ in host_out]),
            ([torch.empty_like(d_) for _, d_ in host_in], [torch.empty_like(d_) for _, d_ in host_out])]
    s_cmp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_e2e(n):
        """n pipelined end-to-end steps; returns the device time of all of them (ms)."""
        ev = lambda: torch.cuda.Event(enable_timing=True)
        in_done, cmp_done, out_done = ([ev() for _ in range(n)] for _ in range(3))
        start, stop = ev(), ev()
        start.record(s_cmp)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            ins, outs = sets[i % 2]
            if i >= 2:
                s_in.wait_event(cmp_done[i - 2])    # the compute of step i - 2 read these inputs
            with torch.cuda.stream(s_in):
                for (h, _), d_ in zip(host_in, ins):
                    d_.copy_(h, non_blocking=True)
            in_done[i].record(s_in)
            s_cmp.wait_event(in_done[i])
            if i >= 2:
                s_cmp.wait_event(out_done[i - 2])   # step i - 2's output has left these buffers
            call(ins, outs)
            cmp_done[i].record(s_cmp)
            s_out.wait_event(cmp_done[i])
            with torch.cuda.stream(s_out):
                for (h, _), d_ in zip(host_out, outs):
                    h.copy_(d_, non_blocking=True)
            out_done[i].record(s_out)
        stop.record(s_out)
        s_cmp.wait_event(stop)
        stop.synchronize()
        return start.elapsed_time(stop)

    for _ in range(args.warmup):
        step()
    run_e2e(2)
    step_full()
    torch.cuda.synchronize()
    assert basa.get_status() == 0, "device wait timed out during warm-up"

    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_steps = time_steps(step, args.steps, flush)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = sum(t_steps) / len(t_steps)
    ms_max = max_over_ranks(ms, world)

    # the step's kernels on their own: pooling into the workspace, then the
    # attention kernel on the pooled tokens (only for workloads with global memory)
    ms_attn, ms_pool = ms_max, 0.0
    if w.P:
        kpt, vpt = basa.pool_kv(dk, dv, w.pool)
        t_pool = time_steps(lambda: basa.pool_kv(dk, dv, w.pool, out=(kpt, vpt)), args.steps,
                            flush)
        t_attn = time_steps(lambda: basa.window_attn_gm(dq, dk, dv, kpt, vpt, w.window, shift,
                                                        w.pool, out=out), args.steps, flush)
        ms_pool = max_over_ranks(sum(t_pool) / len(t_pool), world)
        ms_attn = max_over_ranks(sum(t_attn) / len(t_attn), world)

    # every block of a multi-block shift schedule (FLUX's alternating (0, 0) /
    # (8, 8) blocks; the four shifts of the pooled schedule): each block's own
    # inputs, pooling, attention and pooling + attention, and the schedule's
    # total (the sum of the blocks' steps)
    blocks_out = None
    if len(w.shifts) > 1 and not L and not args.no_blocks:
        blocks_out = []
        for bi, bshift in enumerate(w.shifts):
            bq, bk, bv = (x.to(dev) for x in workload_inputs(w, bi))
            row = {"block": bi, "shift": list(bshift)}
            if w.P:
                bkp, bvp = basa.pool_kv(bk, bv, w.pool)
                tp = time_steps(lambda: basa.pool_kv(bk, bv, w.pool, out=(bkp, bvp)), args.steps,
                                flush)
                ta = time_steps(lambda: basa.window_attn_gm(bq, bk, bv, bkp, bvp, w.window, bshift,
                                                            w.pool, out=out), args.steps, flush)
                row["pool_ms"] = max_over_ranks(sum(tp) / len(tp), world)
                row["attn_ms"] = max_over_ranks(sum(ta) / len(ta), world)
            ts = time_steps(lambda: basa.window_attn(bq, bk, bv, w.window, bshift, w.pool, out=out,
                                                     workspace=ws if ws_bytes else None),
                            args.steps, flush)
            row["step_ms"] = max_over_ranks(sum(ts) / len(ts), world)
            blocks_out.append(row)
            del bq, bk, bv
        assert basa.get_status() == 0, "device wait timed out during the block timings"

    # full attention on the same inputs: the speedup denominator
    t_full = time_steps(step_full, args.full_steps, flush)
    ms_full = max_over_ranks(sum(t_full) / len(t_full), world)

    # context: torch SDPA (opaque library kernels, not this library) on the same
    # inputs, as full attention and as the roll + reshape + SDPA window route
    comparators = None
    if dq.dtype == torch.bfloat16 and not w.P and not L and not args.no_comparators:
        comparators = sdpa_comparators(dq, dk, dv, w, shift, args.full_steps, flush, world)
        if comparators:
            ref = sdpa_window_attn(dq, dk, dv, w.window, shift)
            basa.window_attn(dq, dk, dv, w.window, shift, w.pool, out=out)
            comparators["max_abs_diff_vs_window_route"] = float((out.float() - ref.float()).abs().max())
            del ref

    # end to end through the public API with host buffers (inputs larger than L2
    # arrive from the host every step)
    flush()
    e2e = max_over_ranks(run_e2e(args.steps) / args.steps, world)
    assert basa.get_status() == 0, "device wait timed out during timing"

    peaks = _peaks()
    tflops = world * flops / (ms_max * 1e-3) / 1e12
    per_gpu_tflops = flops / (ms_max * 1e-3) / 1e12
    attn_tflops = flops / (ms_attn * 1e-3) / 1e12   # the attention kernel alone
    gbs = bytes_ / (ms_attn * 1e-3) / 1e9
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / bytes_ >= ridge:   # arithmetic intensity above the ridge point
        roof = {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"]}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof["peak_source"] = peaks["source"]
    kname = "tc_attn_kernel"
    roof["traffic"] = _traffic(kname, w.name)
    roof["kernel"] = kname
    roof["kernel_ms"] = ms_attn

    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic",
        "config": arm_config(w, shift, world),
        "latency_ms": ms_max,
        # this rank's spread over the timed steps (the mean is latency_ms)
        "latency_pct_ms": {"p10": float(np.percentile(t_steps, 10)),
                           "p50": float(np.percentile(t_steps, 50)),
                           "p90": float(np.percentile(t_steps, 90))},
        "pct_bf16_peak": 100.0 * per_gpu_tflops / peaks["bf16_tflops"],
        "speedup": {"full_attn_ms": ms_full, "window_attn_ms": ms_max,
                    "realised": ms_full / ms_max, "theoretical": theo,
                    "ratio": (ms_full / ms_max) / theo,
                    "full_attn_tflops": 4.0 * w.B * w.H * (N + L) ** 2 * w.d / (ms_full * 1e-3) / 1e12},
        "roofline": roof,
        **({"comparators": comparators} if comparators else {}),
        "e2e": {"value": world * flops / (e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e,
                "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h, _ in host_in),
                "d2h_bytes_per_step": sum(h.numel() * h.element_size() for h, _ in host_out),
                "pipeline": "two device buffer sets; copy-in, compute and copy-out streams"},
        "kernels_ms": {kname: ms_attn, "pool_kernel": ms_pool},
        "gpu_launches": args.steps * (2 if (w.P or L) else 1),
        "clocks": clk,
    }
    if blocks_out:
        line["blocks"] = blocks_out
        line["all_blocks_ms"] = sum(r["step_ms"] for r in blocks_out)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, shift, q, k, v)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
