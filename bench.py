#!/usr/bin/env python
"""KDA benchmark: chunked prefill (tokens/s, TFLOP/s vs the bf16 tensor-core
peak) and serving decode (state GB/s vs HBM), one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one prefill of the 8K-token, 32-head, d=128 bf16 workload (fp32
state, chunk 64), inputs resident in HBM. The decode leg runs the 256-sequence
x 32-head serving workload for 1000 one-token steps. With N > 1 (torchrun) every
rank runs its own replica (the work is independent per sequence and head, so
there is no collective on the data path); `value` is the job total.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "bf16_h32_t8192_d128"
DECODE = "decode_n256_h32_d128"
C = 64


def prefill_flops_per_token_head(dk: int, dv: int, chunk: int = C) -> float:
    """Algorithmic FLOPs of the chunked form per (token, head):
    2C(3dk + 2dv) + 6 dk dv + C^2/3 (Gram products, WY apply, state pass, inverse)."""
    return 2 * chunk * (3 * dk + 2 * dv) + 6 * dk * dv + chunk * chunk / 3


def backward_flops_per_token_head(dk: int, dv: int, chunk: int = C) -> float:
    """Algorithmic FLOPs of the chunked backward per (token, head), counting the products
    of its formulas as dense: 2 (7 dk dv + 7 C dk + 5 C dv + 7 C^2 / 3) (seven d_k x d_v
    products such as K~ S, Q~^T dO, dO S^T; seven C x C x d_k ones such as K~ K^^T, dP K^;
    five C x C x d_v ones such as T Y, dU Y^T; the inverse and dA = -N^T dN N^T)."""
    return 2 * (7 * dk * dv + 7 * chunk * dk + 5 * chunk * dv + 7 * chunk * chunk / 3)


def fp32_alu_peak_tflops(sms: int = 148, lanes: int = 128, ghz: float = 1.965) -> float:
    """fp32 FMA peak of the CUDA cores: SMs x fp32 lanes per SM x 2 FLOP x max clock."""
    return round(sms * lanes * 2 * ghz / 1e3, 1)


def prefill_bytes_per_token_head(dk: int, dv: int, elem: int = 2) -> int:
    """Compulsory HBM bytes per (token, head): read q, k, g, v, beta; write out."""
    return elem * (3 * dk + dv + 1) + elem * dv


def measured_traffic(key: str) -> int | None:
    """DRAM bytes per launch from the committed ncu capture, while the kernel source
    that was captured is unchanged (sha256 prefix); otherwise None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[key]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != rec["sha256_16"]:
                return None
        return int(rec.get("bytes_per_call") or rec.get("bytes_per_launch"))
    except (OSError, KeyError, ValueError):
        return None


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """SM clock and throttle-reason sampling (NVML, read-only) during the timed region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int, period_s: float = 0.0005):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None

    def start(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:  # noqa: BLE001 -- no NVML: no clock record
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, bit in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
                except Exception:  # noqa: BLE001
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        t0 = time.time()  # the first sample before any timed work
        while not self.samples and time.time() - t0 < 1.0:
            time.sleep(0.001)

    def mark(self) -> int:
        """Index of the next sample: summary(since=mark()) covers what follows."""
        return len(self.samples)

    def summary(self, since: int = 0) -> dict | None:
        xs = self.samples[since:]
        if not xs:
            return None
        return {"sm_mhz": statistics.median(xs), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(xs)}

    def stop(self) -> dict | None:
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join()
        return self.summary()


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Slowest rank's time: every rank's device time, reduced with MAX."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every replica processes its own tokens each step, and the
    step takes as long as the slowest rank."""
    return tokens_per_rank_step * world / (ms_per_step / 1e3)


def time_region(fn, steps: int, stream) -> tuple[float, list[float]]:
    """Total and per-step device time (ms) of `steps` calls, CUDA events on `stream`."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(steps):
        fn()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    return evs[0].elapsed_time(evs[-1]), per


def bench_ours(args, world, rank, local):
    from kimi_delta_attention_19_b200 import kda
    from kimi_delta_attention_19_b200.inputs import (WORKLOADS, decode_state, decode_tokens,
                                                      workload_inputs)
    peaks = load_peaks()
    dev = f"cuda:{local}"
    stream = torch.cuda.current_stream()
    w = WORKLOADS[PREFILL]
    x = workload_inputs(w, seed=rank, device=dev)
    T, H, dk, dv = w.T, w.H, w.dk, w.dv
    shape = kda.make_shape(T, H, dk, dv, w.dtype)
    ws = kda.alloc_workspace(shape, dev)
    out = torch.empty(T, H, dv, dtype=w.dtype, device=dev)
    fin = torch.empty(1, H, dk, dv, dtype=torch.float32, device=dev)

    def step():
        kda.chunk_fwd(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state, out=out,
                      final_state=fin, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # one sampler (0.5 ms period) over every timed leg below: `clocks` in the line covers
    # all of them, `clocks_prefill_region` the headline prefill's timed region alone
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    mark = clocks.mark()
    total_ms, per = time_region(step, args.steps, stream)
    barrier(world)
    torch.cuda.synchronize()
    clk = clocks.summary(mark)
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    tokens_per_step = T * world
    value = job_tokens_per_s(T, world, ms_step)
    flops = prefill_flops_per_token_head(dk, dv) * T * H
    kernel_ms = statistics.mean(per)
    launches_per_step = kda_launches_per_step(kda, shape)

    tc_tflops = flops / (kernel_ms / 1e3) / 1e12
    algo_bytes = prefill_bytes_per_token_head(dk, dv) * T * H + 2 * 4 * H * dk * dv
    gbs = algo_bytes / (kernel_ms / 1e3) / 1e9
    roofline = {"bound": "tensor", "achieved": round(tc_tflops, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tc_tflops / peaks["bf16_tflops"], 4),
                # the library picks the streamed schedule for this workload (its two kernels run
                # together): its DRAM bytes come from an ncu capture of one whole call inside a
                # profiler range (application-range replay, nothing serialized); the segmented
                # schedule's from a per-kernel capture
                "traffic": (measured_traffic("prefill_bf16_h32_t8192_d128_segmented")
                            if os.environ.get("KDA_PREFILL_SCHEDULE") == "segmented"
                            else measured_traffic("prefill_bf16_h32_t8192_d128")),
                "traffic_segmented_schedule": measured_traffic("prefill_bf16_h32_t8192_d128_segmented"),
                "traffic_scope": "one kda_chunk_fwd call (intra-chunk kernel + walk kernel)",
                "schedule": os.environ.get("KDA_PREFILL_SCHEDULE") or "library model (streamed here)",
                "peak_source": peaks["source"],
                "hbm": {"achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(gbs / peaks["hbm_gbs"], 4), "algo_bytes": algo_bytes},
                "kernel_ms": round(kernel_ms, 4)}

    # ---- end to end through the public API with host buffers. Consecutive steps are
    #      pipelined over three streams (copy in, compute, copy out) with two sets of device
    #      buffers, so one step's read-back overlaps the next step's upload on the two PCIe
    #      directions; every step's own host->device copies and device->host read stay in
    #      the timed region, which runs from the first upload to the last read-back.
    pin = {n: getattr(x, n).cpu().pin_memory() for n in ("q", "k", "v", "g", "beta")}
    s0_host = x.initial_state.cpu().pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    fin_host = [torch.empty(fin.shape, dtype=fin.dtype).pin_memory() for _ in range(2)]
    dbuf = [{n: torch.empty_like(getattr(x, n)) for n in pin} for _ in range(2)]
    s0_dev = [torch.empty_like(x.initial_state) for _ in range(2)]
    out_dev = [out, torch.empty_like(out)]
    fin_dev = [fin, torch.empty_like(fin)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer set b uploaded
    ev_c = [torch.cuda.Event() for _ in range(2)]     # compute on set b done
    ev_out = [torch.cuda.Event() for _ in range(2)]   # outputs of set b read back
    started = [False, False]

    def e2e_step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev_c[b])  # the previous compute on set b has read its inputs
            for n in pin:
                dbuf[b][n].copy_(pin[n], non_blocking=True)
            s0_dev[b].copy_(s0_host, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if started[b]:
            stream.wait_event(ev_out[b])  # the previous read-back of set b is done
        kda.chunk_fwd(dbuf[b]["q"], dbuf[b]["k"], dbuf[b]["v"], dbuf[b]["g"], dbuf[b]["beta"],
                      initial_state=s0_dev[b], out=out_dev[b], final_state=fin_dev[b],
                      workspace=ws, stream=stream)
        ev_c[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            fin_host[b].copy_(fin_dev[b], non_blocking=True)
            ev_out[b].record(s_out)
        started[b] = True

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    n_e2e = max(4, args.steps // 4)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    s_in.wait_event(ev_out[(n_e2e - 1) & 1])
    s_in.wait_event(ev_out[n_e2e & 1])
    t_end.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t_start.elapsed_time(t_end), world) / n_e2e
    h2d = sum(t.numel() * t.element_size() for t in pin.values()) + s0_host.numel() * 4
    d2h = out_host[0].numel() * out_host[0].element_size() + fin_host[0].numel() * 4
    e2e = {"value": round(tokens_per_step / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
           "pipelining": "copy-in, compute and copy-out streams, two buffer sets"}
    del pin, dbuf, s0_dev, out_dev, fin_dev

    # ---- decode leg
    wd = WORKLOADS[DECODE]
    N, Hd, d = wd.B, wd.H, wd.dk
    dsteps = wd.extra["steps"]
    state = decode_state(N, Hd, d, d, seed=rank, device=dev)
    tok = decode_tokens(dsteps, N, Hd, d, d, seed=1000 + rank, device=dev)
    dout = torch.empty(N, Hd, d, dtype=torch.bfloat16, device=dev)

    def dstep(t):
        kda.decode_step(tok.q[t], tok.k[t], tok.v[t], tok.g[t], tok.beta[t], state, out=dout,
                        stream=stream)

    for t in range(3):
        dstep(t)
    torch.cuda.synchronize()
    barrier(world)
    it = iter(range(dsteps))
    d_total, d_per = time_region(lambda: dstep(next(it)), dsteps, stream)
    d_total = max_over_ranks(d_total, world)
    d_ms = d_total / dsteps
    state_bytes = 2 * N * Hd * d * d * 4
    tok_bytes = N * Hd * (3 * d + d + 1) * 2 + N * Hd * d * 2
    d_gbs = (state_bytes + tok_bytes) / (d_ms / 1e3) / 1e9
    decode = {"workload": DECODE, "steps": dsteps, "ms_per_step": round(d_ms, 5),
              "launch": "eager: one kda_decode_step per step, no CUDA graph",
              "state_gbs": round(d_gbs * world, 1), "unit": "GB/s",
              "tokens_per_s": round(N * world / (d_ms / 1e3), 1),
              "roofline": {"bound": "hbm", "achieved": round(d_gbs, 1), "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": round(d_gbs / peaks["hbm_gbs"], 4),
                           "frac_of_8tbs": round(d_gbs / 8000.0, 4),
                           "bytes_per_step": state_bytes + tok_bytes,
                           "traffic": measured_traffic("decode_n256_h32_d128")},
              "gpu_launches": dsteps}
    # ---- backward leg (kda_chunk_bwd on the prefill workload; CUDA-core fp32)
    d_out = torch.randn(x.v.shape, generator=torch.Generator(device=dev).manual_seed(7),
                        device=dev).to(w.dtype)
    bws = torch.empty(int(kda.lib.kda_chunk_bwd_workspace_size(kda.ctypes.byref(shape))),
                      dtype=torch.uint8, device=dev)
    grads = [torch.empty_like(t) for t in (x.q, x.k, x.v, x.g, x.beta)]
    ds0 = torch.empty_like(x.initial_state)

    def bstep():
        rc = kda.lib.kda_chunk_bwd(
            *(kda._ptr(t) for t in (x.q, x.k, x.v, x.g, x.beta, x.initial_state)), None,
            kda._ptr(d_out), None, *(kda._ptr(t) for t in grads), kda._ptr(ds0),
            kda.ctypes.byref(shape), kda._ptr(bws), bws.numel(), kda._stream(stream))
        assert rc == kda.KDA_OK, rc

    for _ in range(3):
        bstep()
    torch.cuda.synchronize()
    barrier(world)
    bsteps = 5
    b_total, _ = time_region(bstep, bsteps, stream)
    b_ms = max_over_ranks(b_total, world) / bsteps
    b_flops = (backward_flops_per_token_head(dk, dv) + prefill_flops_per_token_head(dk, dv)) * T * H
    b_tf = b_flops / (b_ms / 1e3) / 1e12
    fp32_peak = fp32_alu_peak_tflops()
    backward = {"workload": PREFILL, "ms_per_call": round(b_ms, 3),
                "tokens_per_s": round(T * world / (b_ms / 1e3), 1),
                "roofline": {"bound": "alu", "achieved": round(b_tf, 2), "peak": fp32_peak,
                             "unit": "TFLOP/s", "frac": round(b_tf / fp32_peak, 4),
                             "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz",
                             "flops_per_call": b_flops,
                             "traffic": measured_traffic("backward_bf16_h32_t8192_d128"),
                             "traffic_scope": "the bwd_simt_kernel launch of one call"},
                "gpu_launches": bsteps * (kda_launches_per_step(kda, shape) + 5)}
    del bws, grads, x, ws, out, fin
    torch.cuda.empty_cache()
    # ---- the other two prefill workloads beside the 8K one: one long sequence, and
    #      packed variable-length sequences (device-resident inputs, CUDA events)
    others = {}
    for name, reps in (("bf16_h16_t1m_d128", 3), ("varlen8_h32_d128", 5)):
        others[name] = bench_prefill_workload(kda, WORKLOADS[name], reps, world, rank, dev,
                                              stream, peaks)
        torch.cuda.empty_cache()
    clk_all = clocks.stop()
    return {
        "value": round(value, 1), "ms_per_step": round(ms_step, 4),
        "clocks": clk_all if clk_all is not None else clk, "clocks_prefill_region": clk,
        "roofline": roofline, "e2e": e2e, "decode": decode, "backward": backward,
        "prefill_1m": others["bf16_h16_t1m_d128"], "prefill_varlen": others["varlen8_h32_d128"],
        "gpu_launches": launches_per_step * args.steps,
        "tflops": round(tc_tflops * world, 2),
    }


def bench_prefill_workload(kda, w, reps: int, world: int, rank: int, dev: str, stream,
                           peaks: dict) -> dict:
    """kda_chunk_fwd on workload `w` (inputs drawn on the device, one workspace), one
    untimed call then `reps` timed ones; tokens/s, algorithmic TFLOP/s and the fraction
    of the measured bf16 peak, like the headline line."""
    from kimi_delta_attention_19_b200.inputs import workload_inputs
    x = workload_inputs(w, seed=rank, device=dev)
    T_total, H, dk, dv = x.q.shape[0], w.H, w.dk, w.dv
    n = len(x.lengths)
    varlen = x.cu_seqlens is not None
    shape = kda.make_shape(T_total, H, dk, dv, w.dtype, n_seqs=n if varlen else 0,
                           max_seqlen=max(x.lengths) if varlen else 0)
    ws = kda.alloc_workspace(shape, dev)
    out = torch.empty(T_total, H, dv, dtype=w.dtype, device=dev)
    fin = torch.empty(n, H, dk, dv, dtype=torch.float32, device=dev)

    def call():
        kda.chunk_fwd(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state,
                      cu_seqlens=x.cu_seqlens, max_seqlen=max(x.lengths) if varlen else 0,
                      out=out, final_state=fin, workspace=ws, stream=stream)

    call()
    torch.cuda.synchronize()
    barrier(world)
    total, _ = time_region(call, reps, stream)
    ms = max_over_ranks(total, world) / reps
    flops = prefill_flops_per_token_head(dk, dv) * T_total * H
    tf = flops / (ms / 1e3) / 1e12
    algo_bytes = prefill_bytes_per_token_head(dk, dv) * T_total * H + 2 * 4 * n * H * dk * dv
    gbs = algo_bytes / (ms / 1e3) / 1e9
    res = {"workload": w.name, "tokens": T_total, "sequences": n, "heads": H,
           "ms_per_call": round(ms, 4), "calls_timed": reps,
           "tokens_per_s": round(T_total * world / (ms / 1e3), 1),
           "tflops": round(tf * world, 2),
           "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"],
                        "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                        "peak_source": peaks["source"],
                        "hbm": {"achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4)}},
           "gpu_launches": reps * kda_launches_per_step(kda, shape)}
    del x, ws, out, fin
    return res


def kda_launches_per_step(kda, shape) -> int:
    """Kernels one kda_chunk_fwd enqueues for `shape` (the header memset excluded).

    bf16 with d_k = d_v = 128 takes the tensor-core path: the intra-chunk kernel and the
    walk kernel (summary walks, combine steps and output walks of every segment in one
    launch). Other shapes run one CUDA-core kernel."""
    T_total = shape.T * (1 if shape.n_seqs > 0 else shape.B)
    if not (shape.dtype == kda.KDA_BF16 and shape.dk == 128 and shape.dv == 128 and T_total > 0):
        return 1
    return 2


def cpu_oracle_rate(min_seconds: float = 10.0, tokens: int | None = None, seed: int = 0) -> dict:
    """Time the fp64 oracle on the prefill workload's tokens (all heads), repeating
    whole passes until at least `min_seconds` of CPU work has been timed."""
    from kimi_delta_attention_19_b200.inputs import WORKLOADS, workload_inputs
    from oracle import kda_oracle as ko
    w = WORKLOADS[PREFILL]
    x = workload_inputs(w, seed=seed, device="cpu")
    tokens = w.T if tokens is None else min(tokens, w.T)
    sl = slice(0, tokens)
    threads = min(os.cpu_count() or 1, w.H)
    ko.load()
    done, dt = 0, 0.0
    while dt < min_seconds or done == 0:
        t0 = time.perf_counter()
        ko.recurrent(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl],
                     initial_state=x.initial_state, n_threads=threads)
        dt += time.perf_counter() - t0
        done += tokens
    return {"value": round(done / dt, 2), "unit": "tokens/s", "cores": threads,
            "host_cores": os.cpu_count(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"{done // tokens} pass(es) over {tokens} of {w.T} tokens of {PREFILL} "
                      f"(all {w.H} heads), fp64 token-by-token recurrence, {threads} threads"}


def kernels_only(args):
    """Profiler driver: `warmup + steps` calls of one path on its benchmark workload on
    cuda:0 (prefill: kda_chunk_fwd on the 8K x 32-head inputs with one workspace; backward:
    kda_chunk_bwd on the same inputs; decode: chained decode steps on the 256 x 32-head
    state), no timing and no CPU leg. ncu captures select launches with -s/-c on this run."""
    from kimi_delta_attention_19_b200 import kda
    from kimi_delta_attention_19_b200.inputs import (WORKLOADS, decode_state, decode_tokens,
                                                      workload_inputs)
    dev = "cuda:0"
    n = args.warmup + args.steps
    if args.kernels_only == "backward":
        w = WORKLOADS[PREFILL]
        x = workload_inputs(w, device=dev)
        d_out = torch.randn(x.v.shape, generator=torch.Generator(device=dev).manual_seed(7),
                            device=dev).to(w.dtype)
        for _ in range(n):
            kda.chunk_bwd(x.q, x.k, x.v, x.g, x.beta, d_out, initial_state=x.initial_state)
    elif args.kernels_only == "prefill":
        w = WORKLOADS[PREFILL]
        x = workload_inputs(w, device=dev)
        shape = kda.make_shape(w.T, w.H, w.dk, w.dv, w.dtype)
        ws = kda.alloc_workspace(shape, dev)
        for i in range(n):
            # --profile-range: the last call inside a profiler range (cudaProfilerStart/Stop),
            # for a range-replay capture that keeps the call's two kernels running together
            last = args.profile_range and i == n - 1
            if last:
                torch.cuda.synchronize()
                torch.cuda.cudart().cudaProfilerStart()
            kda.chunk_fwd(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state,
                          workspace=ws)
            if last:
                torch.cuda.synchronize()
                torch.cuda.cudart().cudaProfilerStop()
    else:
        wd = WORKLOADS[DECODE]
        state = decode_state(wd.B, wd.H, wd.dk, wd.dv, device=dev)
        tok = decode_tokens(n, wd.B, wd.H, wd.dk, wd.dv, seed=1000, device=dev)
        for t in range(n):
            kda.decode_step(tok.q[t], tok.k[t], tok.v[t], tok.g[t], tok.beta[t], state)
    torch.cuda.synchronize()
    print(f"kernels-only {args.kernels_only}: {n} calls done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=2048,
                    help="tokens per reference-arm step (bounded oracle sample)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="minimum timed oracle work for the cpu_baseline object")
    ap.add_argument("--profile-range", action="store_true",
                    help="with --kernels-only prefill: put the last call inside a profiler range")
    ap.add_argument("--kernels-only", choices=["prefill", "backward", "decode"], default=None,
                    help="profiler driver: run warmup + steps calls of one path, print no "
                         "measurement (for ncu -s/-c captures)")
    args = ap.parse_args()
    if args.kernels_only:
        kernels_only(args)
        return
    args.warmup = max(args.warmup, 3)
    cfg = {"workload": PREFILL, "model": "KDA layer (synthetic, no weights)", "global_batch": 1,
           "seq_len": 8192, "heads": 32, "dk": 128, "dv": 128, "chunk": C,
           "state": "fp32", "l2": "inputs_exceed_l2 (q,k,v,g 256 MiB > 126 MB L2)"}
    metric = "KDA prefill tokens/s + % bf16 TC peak; decode state GB/s vs HBM peak"

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        cfg["parallelism"] = f"oracle on host cores (N={world} requested; rank 0 only)"
        rates = []
        cpu_oracle_rate(min_seconds=0.0, tokens=256)  # warm-up (library load, page-in)
        for _ in range(args.steps):
            rates.append(cpu_oracle_rate(min_seconds=0.0, tokens=args.cpu_tokens))
        v = statistics.median(r["value"] for r in rates)
        cb = dict(rates[-1])
        cb["value"] = v
        print(json.dumps({
            "metric": metric, "value": v, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * args.cpu_tokens / v, 3) if v else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg, "impl": "reference", "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    world, rank, local = dist_setup(args.gpus)
    cfg["parallelism"] = f"replicas{world}" if world > 1 else "single_gpu"
    r = bench_ours(args, world, rank, local)
    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_oracle_rate(min_seconds=args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": metric, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded; no weights, no dataset)",
            "config": cfg, "impl": "ours", "tflops": r["tflops"], "roofline": r["roofline"],
            "cpu_baseline": cpu, "e2e": r["e2e"], "gpu_launches": r["gpu_launches"],
            "clocks": r["clocks"], "clocks_prefill_region": r["clocks_prefill_region"],
            "decode": r["decode"], "backward": r["backward"],
            "prefill_1m": r["prefill_1m"], "prefill_varlen": r["prefill_varlen"],
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
