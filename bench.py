"""Benchmark of the attention hot path on B200.

Headline workload (one GPU): the 128K long-context prefill, B=1, S=131072,
Hq=32, Hkv=8, D=128, bf16, one causal document (the largest single-GPU
workload). One step is one llama_attn_prefill call over that batch (K
rotation, tensor-core attention). The metric counts only unmasked (i, j)
pairs: FLOPs = 4 * D * Hq * pairs. In the same run the other prefill
workloads (8B-shaped packed, B=4, S=8192, Hq=32, documents U[512, 4096];
405B-shaped, B=1, S=16384, Hq=128, documents U[1024, 8192]) are timed the same
way and reported under "prefill_workloads", each with its own roofline, end to
end figure and CPU baseline; the decode form (70B-shaped, 64 sequences, Hq=64,
Hkv=8, cache lengths U[1024, 32768]) is reported under "decode" (GB/s of cached
K/V rows read).

`--impl reference` times the float64 CPU oracle on the host cores instead, on
a bounded sample of query rows of the same workload, in the same unit.

Multi-GPU (torchrun): by default one process per GPU, each with its own
independent batch (weak scaling, no data-path collective); rank 0 prints the
line, value = FLOPs of all ranks / max-over-ranks time.

Also timed by default: the headline prefill with its LSE output and KV-cache
append (`prefill_ex`), and the FP8 E4M3 QKV projection with RoPE on the 8B
packed workload's tokens (`qkv_fp8`).

Options:
  --shard kv-groups  one workload split over the GPUs by KV group (each rank
                     its Hkv/N KV heads and their query heads; strong scaling)
  --cp               context-parallel prefill of one single-document workload
                     over the GPUs (zigzag split, K/V all-gather, strong scaling)
  --decode-page-size the decode through the paged-cache entry point
  --no-prefill-ex, --no-qkv-fp8, --no-decode, --no-extra  skip those measurements
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gqa_attention_rope_b200 import workloads as W  # noqa: E402

METRIC = "prefill attention TFLOP/s (causal) & decode KV-cache GB/s, % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, "measured" or
    "fallback"): the measured copy bandwidth and cuBLAS bf16 throughput of this
    pool's B200s, else the earlier pool measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        burst = float(pk["bf16_tflops"])
        return float(pk["hbm_gbs"]), burst, float(pk.get("bf16_tflops_sustained") or burst), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# A kernel timed for longer than this in one timed region runs at the power
# cap's sustained clock, so it is compared with the sustained tensor peak.
SUSTAINED_AFTER_S = 1.0


class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms through NVML (in a
    thread) while the timed region runs; without NVML the record says so."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.reasons = set()
        self._stop = None
        self._thread = None
        self.max_mhz = None

    def _handle(self):
        """NVML handle of this process's CUDA device, found by its PCI address
        (CUDA and NVML may number devices differently)."""
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.cuda_index)
        dom, bus, dev = (getattr(props, n, None) for n in ("pci_domain_id", "pci_bus_id", "pci_device_id"))
        if all(isinstance(x, int) for x in (dom, bus, dev)):
            return pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08X}:{bus:02X}:{dev:02X}.0".encode())
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._thread = None
            return
        self._stop = threading.Event()

        def run():
            get_r = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    bits = get_r(h)
                    for b, n in self.REASONS.items():
                        if bits & b:
                            self.reasons.add(n)
                except Exception:
                    pass
                self._stop.wait(0.005)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        self._stop.set()
        self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- CPU oracle baseline

def oracle_rows_sample(w, inp, target_s: float, seed: int = 99):
    """Time the float64 oracle on growing samples of query rows until about
    target_s seconds of work; returns (flops_done, seconds, n_rows, threads)."""
    from oracle import oracle as O
    lay = O.doc_layout(inp["doc_offsets"], w.B, w.S)
    ds = lay[0].astype(np.int64)
    g = np.random.default_rng(seed)
    n = 8
    while True:
        rows = np.sort(g.choice(w.B * w.S, size=n, replace=False))
        t0 = time.perf_counter()
        O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"], w.rope_theta, rows=rows, layout=lay)
        dt = time.perf_counter() - t0
        visible = ((rows % w.S) - ds[rows] + 1).sum()  # keys each sampled row attends to
        flops = 4.0 * w.D * w.Hq * float(visible)
        if dt >= target_s or n >= w.B * w.S // 2:
            return flops, dt, n, O.num_threads()
        n = int(min(w.B * w.S // 2, max(2 * n, n * target_s / max(dt, 1e-3))))


def run_reference(args, w):
    """The oracle as the reference arm: each step is a bounded sample of rows."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = W.make_prefill_inputs(w)
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_rows_sample(w, inp, per_step / 4)
    flops = secs = 0.0
    rows = threads = 0
    for _ in range(args.steps):
        f, s, n, threads = oracle_rows_sample(w, inp, per_step)
        flops += f
        secs += s
        rows += n
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} random query rows x {w.Hq} heads of {w.name} over {args.steps} steps "
                                   "(float64 C oracle, OpenMP, full masked rows)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, world, shard="replicas"):
    if world == 1:
        par = "1 GPU"
    elif shard == "kv-groups":
        par = f"one workload split by KV group over {world} GPUs ({w.Hkv // world} KV heads per GPU; strong scaling)"
    else:
        par = f"{world} independent replicas (weak scaling)"
    return {"workload": w.name, "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "doc_lengths": None if w.doc_range is None else f"U[{w.doc_range[0]},{w.doc_range[1]}]",
            "rope_theta": w.rope_theta, "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
            "parallelism": par}


# ---------------------------------------------------------------- GPU arm

def cpu_baseline_of(w, inp, seconds):
    f, s, n, threads = oracle_rows_sample(w, inp, seconds)
    return {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} random query rows x {w.Hq} heads of {w.name} (float64 C oracle, "
                      f"full masked rows, {s:.1f} s)"}


def measure_prefill(args, la, dev, w, world, rank, peaks, cpu_seconds, steps):
    """Times `steps` prefill steps of workload w on this rank (device time,
    CUDA events, L2 flushed between steps), then the same steps end to end
    through the public API with pinned host buffers. Returns one record."""
    hbm_peak, tc_peak, tc_sust, peak_kind = peaks
    shard = args.shard if world > 1 else "replicas"
    if shard == "kv-groups":
        # the same workload on every rank; this rank's KV groups and their query heads
        from gqa_attention_rope_b200 import kv_group_parallel as KG
        full = W.make_prefill_inputs(w)
        q_h, k_h, v_h = KG.shard_qkv(full["q"], full["k"], full["v"], world, rank)
        inp = dict(q=q_h, k=k_h, v=v_h, doc_offsets=full["doc_offsets"])
        wr = w
        heads_local = q_h.shape[2]
    else:
        wr = W.PrefillWorkload(w.name, w.seed + 1000 * rank, w.B, w.S, w.Hq, w.Hkv, w.D, w.dtype, w.doc_range,
                               w.rope_theta)  # per-rank seed: ranks hold independent batches
        inp = W.make_prefill_inputs(wr)
        heads_local = w.Hq
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    offs = inp["doc_offsets"].to(dev) if inp["doc_offsets"] is not None else None
    out = torch.empty_like(q)
    pairs = W.unmasked_pairs(inp["doc_offsets"], wr.B, wr.S)
    flops = 4.0 * w.D * heads_local * pairs  # this rank's FLOPs per step
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        la.llama_attn_prefill(q, k, v, out=out, doc_offsets=offs, rope_theta=w.rope_theta)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if la.llama_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    clocks = ClockSampler(dev.index)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    la.llama_attn_profile_begin()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    main_ms, main_n, launches = la.llama_attn_profile_end()
    barrier(world)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    all_flops = sum_over_ranks(flops * steps, world)
    value = all_flops / (total_ms / 1e3) / 1e12
    kernel_ms = main_ms / max(main_n, 1)
    achieved = flops / (kernel_ms / 1e3) / 1e12
    sustained = kernel_ms * steps / 1e3 > SUSTAINED_AFTER_S
    peak = tc_sust if sustained else tc_peak

    # End to end through the public API, as a serving loop runs it: every step
    # uploads its own q, k, v (and offsets) from pinned host memory and
    # downloads its output, on two copy streams, with double-buffered device
    # tensors, so the upload of step i+1 and the download of step i-1 overlap
    # the kernels of step i. The timed region runs from the first upload to
    # the last download.
    hq, hk, hv = (inp[n].pin_memory() for n in ("q", "k", "v"))
    hoffs = inp["doc_offsets"].pin_memory() if inp["doc_offsets"] is not None else None
    houts = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    bufs = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), o=torch.empty_like(q),
                 offs=torch.empty_like(offs) if offs is not None else None) for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        up_ev = [torch.cuda.Event() for _ in range(n)]
        comp_ev = [torch.cuda.Event() for _ in range(n)]
        down_ev = [torch.cuda.Event() for _ in range(n)]
        t0.record(stream)
        up.wait_event(t0)
        for i in range(n):
            b = bufs[i % 2]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(comp_ev[i - 2])  # the kernels of step i-2 have read this buffer
                b["q"].copy_(hq, non_blocking=True)
                b["k"].copy_(hk, non_blocking=True)
                b["v"].copy_(hv, non_blocking=True)
                if b["offs"] is not None:
                    b["offs"].copy_(hoffs, non_blocking=True)
                up_ev[i].record(up)
            stream.wait_event(up_ev[i])
            if i >= 2:
                stream.wait_event(down_ev[i - 2])  # step i-2's output has left this buffer
            la.llama_attn_prefill(b["q"], b["k"], b["v"], out=b["o"], doc_offsets=b["offs"],
                                  rope_theta=w.rope_theta, stream=stream)
            comp_ev[i].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(comp_ev[i])
                houts[i % 2].copy_(b["o"], non_blocking=True)
                down_ev[i].record(down)
        stream.wait_event(down_ev[n - 1])
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(3)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_run(steps), world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv)) + (hoffs.numel() * 4 if hoffs is not None else 0)
    d2h = houts[0].numel() * houts[0].element_size()
    e2e = {"value": all_flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / steps,
           "pipeline": "each step uploads its inputs and downloads its output (pinned host memory); "
                       "double-buffered on two copy streams, so step i+1's upload and step i-1's download "
                       "overlap step i's kernels"}
    del bufs, houts
    if la.llama_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during the benchmark")
    cpu = None
    if rank == 0 and world == 1 and cpu_seconds > 0:
        cpu = cpu_baseline_of(wr, inp, cpu_seconds)
    return {
        "workload": w.name, "value": value, "unit": "TFLOP/s", "steps": steps, "ms_per_step": total_ms / steps,
        "flops_per_step_per_gpu": flops, "unmasked_pairs_per_head": pairs,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 dense ({'sustained' if sustained else 'burst'})",
                     "kernel": "prefill_bf16_kernel", "kernel_ms": kernel_ms,
                     "traffic": load_traffic("prefill_bf16_kernel", w.name)},
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "gpu_launches": launches,
        "config": config_of(w, world, shard),
    }


def run_ours(args, w):
    import gqa_attention_rope_b200 as la
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    la.lib()
    peaks = load_peaks()
    if args.shard == "kv-groups" and w.Hkv % world != 0:
        raise SystemExit(f"--shard kv-groups needs the GPU count to divide Hkv = {w.Hkv}")

    head = measure_prefill(args, la, dev, w, world, rank, peaks, 0 if args.no_cpu_baseline else args.cpu_seconds,
                           args.steps)
    extras = {}
    for name in ([] if args.no_extra else [n for n in args.extra_workloads.split(",") if n and n != w.name]):
        wx = W.WORKLOADS[name]
        if args.shard == "kv-groups" and wx.Hkv % world != 0:
            continue
        rec = measure_prefill(args, la, dev, wx, world, rank, peaks,
                              0 if args.no_cpu_baseline else args.extra_cpu_seconds, max(args.steps, 10))
        extras[name] = rec
    hbm_peak, tc_peak, tc_sust, peak_kind = peaks
    decode = None if args.no_decode else run_decode(args, la, dev, world, rank, hbm_peak, peak_kind)
    wr = W.PrefillWorkload(w.name, w.seed + 1000 * rank, w.B, w.S, w.Hq, w.Hkv, w.D, w.dtype, w.doc_range,
                           w.rope_theta)
    qkv = None
    if args.qkv_fp8:  # the 8B packed workload's tokens (d_model 4096), per rank
        w8 = W.PACKED_8B
        w8r = W.PrefillWorkload(w8.name, w8.seed + 1000 * rank, w8.B, w8.S, w8.Hq, w8.Hkv, w8.D, w8.dtype,
                                w8.doc_range, w8.rope_theta)
        qkv = run_qkv_fp8(args, la, dev, w8r, tc_peak, peak_kind)
    pex = run_prefill_ex(args, la, dev, wr, tc_peak, tc_sust, peak_kind) if args.prefill_ex else None
    if la.llama_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during the benchmark")

    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "strong" if (world > 1 and args.shard == "kv-groups") else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(head["config"], flops_per_step_per_gpu=head["flops_per_step_per_gpu"],
                       unmasked_pairs_per_head=head["unmasked_pairs_per_head"]),
        "roofline": head["roofline"],
        "cpu_baseline": head["cpu_baseline"],
        "e2e": head["e2e"],
        "clocks": head["clocks"],
        "gpu_launches": (head["gpu_launches"] + sum(r["gpu_launches"] for r in extras.values())
                         + (decode["gpu_launches"] if decode else 0) + (qkv["gpu_launches"] if qkv else 0)
                         + (pex["gpu_launches"] if pex else 0)),
        "prefill_workloads": {n: {k: r[k] for k in ("value", "unit", "steps", "ms_per_step",
                                                    "flops_per_step_per_gpu", "unmasked_pairs_per_head", "roofline",
                                                    "e2e", "cpu_baseline", "clocks", "gpu_launches", "config")}
                              for n, r in extras.items()},
        "decode": decode,
    }
    if qkv is not None:
        line["qkv_fp8"] = qkv
    if pex is not None:
        line["prefill_ex"] = pex
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_cp(args, w):
    """Context-parallel prefill of one workload over the ranks (strong
    scaling): every rank holds its zigzag shard of q, k and v; a step is the
    K/V all-gather plus the local llama_attn_prefill_cp call."""
    import gqa_attention_rope_b200 as la
    from gqa_attention_rope_b200 import context_parallel as CP
    if w.doc_range is not None:
        raise SystemExit("--cp takes a single-document workload (each batch row one document)")
    world, rank, local = dist_setup(args.gpus)
    group = None
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    la.lib()
    hbm_peak, tc_peak, tc_sust, peak_kind = load_peaks()
    inp = W.make_prefill_inputs(w)  # the same seeded sequence on every rank
    ql, kl, vl = (CP.shard_rows(inp[n], world, rank).to(dev) for n in ("q", "k", "v"))
    pos_a, pos_b, L = CP.zigzag_chunks(w.S, world, rank)
    rows = np.r_[pos_a:pos_a + L, pos_b:pos_b + L]
    flops_local = 4.0 * w.D * w.Hq * w.B * float(np.sum(rows + 1))
    flops_total = 4.0 * w.D * w.Hq * W.unmasked_pairs(None, w.B, w.S)
    out = torch.empty_like(ql)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(q_, k_, v_, o_):
        k_full = CP.gather_sequence(k_, world, group)
        v_full = CP.gather_sequence(v_, world, group)
        la.llama_attn_prefill_cp(q_, k_full, v_full, pos_a, L, pos_b, out=o_, rope_theta=w.rope_theta)

    for _ in range(max(3, args.warmup)):
        step(ql, kl, vl, out)
    torch.cuda.synchronize()
    if la.llama_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    clocks = ClockSampler(local)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    la.llama_attn_profile_begin()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step(ql, kl, vl, out)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    main_ms, main_n, launches = la.llama_attn_profile_end()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world)
    value = flops_total * args.steps / (total_ms / 1e3) / 1e12
    kernel_ms = main_ms / max(main_n, 1)
    achieved = flops_local / (kernel_ms / 1e3) / 1e12
    sustained = kernel_ms * args.steps / 1e3 > SUSTAINED_AFTER_S
    peak = tc_sust if sustained else tc_peak

    # end to end: the rank's pinned host shards in, its output rows back
    hq, hk, hv = (t.cpu().pin_memory() for t in (ql, kl, vl))
    hout = torch.empty(ql.shape, dtype=ql.dtype).pin_memory()
    dq, dk, dv, dout = torch.empty_like(ql), torch.empty_like(kl), torch.empty_like(vl), torch.empty_like(ql)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        step(dq, dk, dv, dout)
        hout.copy_(dout, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    for i in range(args.steps):
        e_ev[i][0].record(stream)
        e2e_step()
        e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev), world)
    if la.llama_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during the benchmark")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, s, n, threads = oracle_rows_sample(w, inp, args.cpu_seconds)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} random query rows x {w.Hq} heads of {w.name} (float64 C oracle, "
                         f"full masked rows, {s:.1f} s)"}
    cfg = config_of(w, world)
    cfg["parallelism"] = (f"context parallel over {world} GPU(s): zigzag split into {2 * world} chunks, "
                          "K/V all-gather (NCCL) into local memory, local kernel")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(cfg, flops_per_step_total=flops_total),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 dense ({'sustained' if sustained else 'burst'})",
                     "kernel": "prefill_bf16_kernel", "kernel_ms": kernel_ms, "traffic": None},
        "cpu_baseline": cpu,
        "e2e": {"value": flops_total * args.steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv)),
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "clocks": clk,
        "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_prefill_ex(args, la, dev, w, tc_peak, tc_sust, peak_kind):
    """The prefill step with its two decode-linking outputs: per-row LSE and the
    append of rotated K and V to a [B, Hkv, S, D] decode-layout cache."""
    inp = W.make_prefill_inputs(w)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    offs = inp["doc_offsets"].to(dev) if inp["doc_offsets"] is not None else None
    flops = 4.0 * w.D * w.Hq * W.unmasked_pairs(inp["doc_offsets"], w.B, w.S)
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.S, w.Hq, dtype=torch.float32, device=dev)
    kc = torch.empty(w.B, w.Hkv, w.S, w.D, dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        la.llama_attn_prefill_ex(q, k, v, out=out, lse=lse, doc_offsets=offs, rope_theta=w.rope_theta,
                                 kcache=kc, vcache=vc)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(args.steps, 10)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    la.llama_attn_profile_begin()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    main_ms, main_n, launches = la.llama_attn_profile_end()
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    kernel_ms = main_ms / max(main_n, 1)
    sustained = kernel_ms * steps / 1e3 > SUSTAINED_AFTER_S
    peak = tc_sust if sustained else tc_peak
    achieved = flops / (kernel_ms / 1e3) / 1e12
    return {
        "workload": w.name + " + lse + kv cache append", "value": flops / (step_ms / 1e3) / 1e12, "unit": "TFLOP/s",
        "steps": steps, "ms_per_step": step_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 dense ({'sustained' if sustained else 'burst'})",
                     "kernel": "prefill_bf16_kernel", "kernel_ms": kernel_ms, "traffic": None},
        "gpu_launches": launches,
    }


def run_qkv_fp8(args, la, dev, w, tc_peak, peak_kind):
    """The FP8 E4M3 QKV projection with RoPE for the prefill workload's tokens
    (d_model = 128 * Hq, the Llama 3 width for these head counts): per step the
    per-tensor quantization of X plus the projection GEMM with its RoPE
    epilogue; the weight is quantized once, outside the timed region."""
    d_model = 128 * w.Hq
    M, N = w.B * w.S, (w.Hq + 2 * w.Hkv) * 128
    g = torch.Generator(device=dev).manual_seed(w.seed + 17)
    x = torch.randn(M, d_model, device=dev, generator=g).to(torch.bfloat16)
    wt = (torch.randn(N, d_model, device=dev, generator=g) * d_model ** -0.5).to(torch.bfloat16)
    inp_offs = W.make_prefill_inputs(w)["doc_offsets"]
    offs = inp_offs.to(dev) if inp_offs is not None else None
    wc, sw = la.llama_attn_quantize_e4m3(wt)
    xc, sx = la.llama_attn_quantize_e4m3(x)
    q = torch.empty(w.B, w.S, w.Hq, 128, dtype=torch.bfloat16, device=dev)
    k = torch.empty(w.B, w.S, w.Hkv, 128, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        la.llama_attn_quantize_e4m3(x, y=xc, scale=sx)
        la.llama_attn_qkv_fp8_rope(xc, sx, wc, sw, w.B, w.S, w.Hq, w.Hkv, doc_offsets=offs,
                                   rope_theta=w.rope_theta, q=q, k=k, v=v)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(args.steps, 10)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    la.llama_attn_profile_begin()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    main_ms, main_n, launches = la.llama_attn_profile_end()
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    flops = 2.0 * M * N * d_model
    kernel_ms = main_ms / max(main_n, 1)
    fp8_peak = 2.0 * tc_peak
    return {
        "workload": f"qkv_fp8_rope_M{M}_K{d_model}_N{N} ({w.name} tokens)", "value": flops / (step_ms / 1e3) / 1e12,
        "unit": "TFLOP/s", "steps": steps, "ms_per_step": step_ms,
        "roofline": {"bound": "tensor", "achieved": flops / (kernel_ms / 1e3) / 1e12, "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": flops / (kernel_ms / 1e3) / 1e12 / fp8_peak,
                     "peak_kind": f"2 x {peak_kind} bf16 dense burst (nominal fp8:bf16 ratio)",
                     "kernel": "qkv_fp8_rope_kernel", "kernel_ms": kernel_ms,
                     "traffic": load_traffic("qkv_fp8_rope_kernel", f"qkv_fp8_rope_M{M}_K{d_model}_N{N}")},
        "gpu_launches": launches,
    }


def run_decode(args, la, dev, world, rank, hbm_peak, peak_kind):
    w = W.DECODE_70B
    nseq = args.decode_seqs
    name = w.name if nseq == w.B else w.name.replace(f"B{w.B}_", f"B{nseq}_")
    w = W.DecodeWorkload(name, w.seed, nseq, w.Hq, w.Hkv, w.D, w.Lmax, w.len_range)
    wr = W.DecodeWorkload(w.name, w.seed + 1000 * rank, w.B, w.Hq, w.Hkv, w.D, w.Lmax, w.len_range)
    inp = W.make_decode_inputs(wr, poison=True)
    q, kc, vc, lens = (inp[n].to(dev) for n in ("q", "kcache", "vcache", "cache_lens"))
    del inp["kcache"], inp["vcache"]
    out = torch.empty_like(q)
    ws = torch.empty(la.llama_attn_decode_workspace_size(w.B, w.Hq, w.Lmax, w.D), dtype=torch.uint8, device=dev)
    tokens = W.cache_tokens(inp["cache_lens"])
    kv_bytes = tokens * w.Hkv * w.D * 2 * 2
    io_bytes = q.numel() * 2 * 2 + lens.numel() * 4
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        la.llama_attn_decode(q, kc, vc, lens, out=out, workspace=ws, rope_theta=w.rope_theta)

    if args.decode_page_size:
        # the same cache rows scattered over a page pool by a fixed permutation
        import ctypes
        P = args.decode_page_size
        max_blocks = (w.Lmax + P - 1) // P
        need = [(int(n) + P - 1) // P for n in inp["cache_lens"]]
        n_pages = sum(need)
        perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(1234)).tolist()
        kp = torch.empty((n_pages, w.Hkv, P, w.D), dtype=torch.bfloat16, device=dev)
        vp = torch.empty_like(kp)
        table = torch.full((w.B, max_blocks), -1, dtype=torch.int32)
        it = iter(perm)
        for b in range(w.B):
            for j in range(need[b]):
                pg = next(it)
                table[b, j] = pg
                lo, hi = j * P, min((j + 1) * P, w.Lmax)
                kp[pg, :, :hi - lo] = kc[b, :, lo:hi]
                vp[pg, :, :hi - lo] = vc[b, :, lo:hi]
        table = table.to(dev)
        del kc, vc
        torch.cuda.empty_cache()
        lib = la.lib()
        sptr = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())

        def step():  # noqa: F811
            st = lib.llama_attn_decode_paged(ptr(q), ptr(kp), ptr(vp), ptr(table), ptr(lens), ptr(out), w.B, w.Hq,
                                             w.Hkv, w.D, P, max_blocks, n_pages, ctypes.c_float(w.rope_theta),
                                             ptr(ws), ws.numel(), sptr)
            assert st == 0

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    steps = max(args.steps, 10)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    la.llama_attn_profile_begin()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    main_ms, main_n, launches = la.llama_attn_profile_end()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world)
    all_bytes = sum_over_ranks(float(kv_bytes + io_bytes) * steps, world)
    kernel_ms = main_ms / max(main_n, 1)
    achieved = kv_bytes / (kernel_ms / 1e3) / 1e9
    return {
        "workload": w.name + (f"_paged{args.decode_page_size}" if args.decode_page_size else ""),
        "value": all_bytes / (total_ms / 1e3) / 1e9, "unit": "GB/s", "steps": steps,
        "ms_per_step": total_ms / steps, "bytes_per_step_per_gpu": kv_bytes + io_bytes, "cache_tokens": tokens,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": f"{peak_kind} HBM copy",
                     "kernel": "decode_split_kernel", "kernel_ms": kernel_ms,
                     "traffic": load_traffic("decode_split_kernel", w.name)},
        "gpu_launches": launches,
    }


def code_sha1(text: str) -> str:
    """sha1 of C/C++/CUDA source with its comments, trailing blanks and empty
    lines removed, so that editing a comment leaves it unchanged while any change
    to the code (including whitespace inside a line) changes it."""
    import hashlib
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or character literal, copied with its escapes
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).split("\n")]
    return hashlib.sha1("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu record, or None when there is
    no record for this kernel and workload or the kernel's code (comments aside)
    has changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel][workload]
        with open(os.path.join(ROOT, rec["source"])) as f:
            if code_sha1(f.read()) != rec["code_sha1"]:
                return None
        return rec["bytes"]
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    prefill_names = [n for n, x in W.WORKLOADS.items() if isinstance(x, W.PrefillWorkload) and x.dtype == "bf16"]
    prefill_names += list(W.CAPTURE_WORKLOADS)  # smaller launches for counter captures only
    ap.add_argument("--workload", default=W.LONG_128K.name, choices=prefill_names,
                    help="the headline prefill workload (the line's value)")
    ap.add_argument("--extra-workloads", default=",".join([W.PACKED_8B.name, W.PACKED_405B.name]),
                    help="comma-separated prefill workloads also timed and reported under prefill_workloads")
    ap.add_argument("--no-extra", action="store_true", help="time the headline workload only")
    ap.add_argument("--extra-cpu-seconds", type=float, default=8.0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "kv-groups"],
                    help="N>1: independent replicas per GPU (weak), or one workload split by KV group (strong)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-seqs", type=int, default=W.DECODE_70B.B,
                    help="sequences in the decode batch (64 = the 70B-shaped workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-page-size", type=int, default=0,
                    help="time the decode through the paged-cache entry point with this page size")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-prefill-ex", dest="prefill_ex", action="store_false",
                    help="skip the prefill with LSE output and KV-cache append (timed by default)")
    ap.add_argument("--no-qkv-fp8", dest="qkv_fp8", action="store_false",
                    help="skip the FP8 QKV projection with RoPE on the 8B packed workload's tokens (timed by default)")
    ap.add_argument("--cp", action="store_true",
                    help="context-parallel prefill of the workload over the GPUs (strong scaling)")
    args = ap.parse_args()
    w = W.WORKLOADS.get(args.workload) or W.CAPTURE_WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        if w.dtype != "bf16":
            raise SystemExit("the bench times the bf16 tensor-core path")
        run_cp(args, w) if args.cp else run_ours(args, w)


if __name__ == "__main__":
    main()
