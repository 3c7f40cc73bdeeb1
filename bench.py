#!/usr/bin/env python
"""Benchmark: FRM image pairs/s at 512x384, d=24 (plus exhaustive MNN pair-scores/s).

One step = Fast Reciprocal Matching of a batch of distinct synthetic image
pairs (512x384, d=24, unit-norm fp16 descriptors, seed stride 8 -> 3072
seeds, max_iter 10) through the batched C-ABI entry point: seed init, 10 x
(NN2 half-step + update, NN1 half-step + update), merge.  The batch's inputs
(8 pairs = 151 MB) exceed the 126 MB L2, so no flush is needed between steps.

Printed: one JSON line (rank 0).  ``value`` = pairs/s over all ranks (each
rank matches its own pairs: weak scaling, no data-path collective), timed on
the device with CUDA events between barriers, max over ranks.  Extra keys:
``e2e`` (host buffers, copies inside the timed region), ``roofline`` (the
fused similarity+argmax kernel, timed live with CUDA events), ``mnn`` (the
exhaustive reciprocal set at 512x384 with its own roofline), ``frm_graph_plan``
(the same step replayed as a recorded graph plan), ``cpu_baseline``
(the double-precision oracle on a bounded sample), ``clocks``,
``gpu_launches``.

``--impl reference`` times the oracle itself (host cores) on the same metric.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of
# the fused kernel in the bench step, from one ncu capture of the step's
# first FRM call (20 launches averaged).  It belongs to the sources that
# determine that kernel's memory traffic (see _kernel_sources_sha256): with any
# other sources the bench reports traffic as null.
TRAFFIC = {"sources_sha256": "c420dfd32bec45cd77db817ca97c9e7fc7813d08cf1aaca6d59ad29529010e7d",
           "frm_nn_bytes_per_launch": 37.23e6}

# What fixes the fused kernel's traffic: its own code and the PTX helpers,
# and in the ABI source the functions that size its tiles, launch it, build
# its tensor maps and write the zero-padded rows it reads.
_TRAFFIC_FILES = ("nn_kernel.cuh", "ptx.cuh")
_TRAFFIC_FUNCS = ("static Geometry geometry(", "static rnn_status launch_nn(",
                  "static rnn_status make_map(", "__device__ __forceinline__ uint4 prep_chunk(",
                  "__global__ void prep_rows_kernel(")


def _kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "reciprocal_nearest_neighbour_b200", "csrc")
    for f in _TRAFFIC_FILES:
        h.update(f.encode())
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "rnn.cu")) as fh:
        text = fh.read()
    for sig in _TRAFFIC_FUNCS:
        i = text.index(sig)
        h.update(text[i:text.index("\n}\n", i)].encode())
    return h.hexdigest()

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("FRM image pairs/s at 512×384, d=24; exhaustive MNN pair-scores/s; "
          "% roofline")
WORKLOAD = "frm_512x384"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


class ClockSampler:
    """SM clock and throttle reasons of one GPU, polled every 5 ms while running.

    Reads NVML (the data nvidia-smi prints); the GPU is matched by UUID so a
    remapped CUDA_VISIBLE_DEVICES does not matter.  Reading changes nothing.
    """

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, device):
        self.device = device
        self.samples = []
        self._stop = None
        self._thread = None
        self._nvml = None
        self._handle = None
        self.max_mhz = None

    def __enter__(self):
        import threading

        import torch

        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception:  # no NVML: clocks are reported as null
            self._nvml = None
            return self
        self._stop = threading.Event()

        def poll():
            nv = self._nvml
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM)
                    mask = get_reasons(self._handle) if get_reasons else 0
                    self.samples.append((mhz, mask))
                except Exception:
                    pass
                self._stop.wait(0.005)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        mx = self.max_mhz or max(m for m, _ in self.samples)
        loaded = [s for s in self.samples if s[0] > 0.5 * mx] or self.samples
        reasons = sorted(name for name, attr in self.REASONS.items()
                         if any(mask & getattr(self._nvml, attr, 0) for _, mask in loaded))
        return {"sm_mhz": statistics.median(m for m, _ in loaded), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def _dist():
    from reciprocal_nearest_neighbour_b200 import replicas
    return replicas.env()


def _oracle_frm_pairs_per_s(maps, budget_s: float, max_pairs: int):
    """Time the oracle's FRM on whole pairs until `budget_s` is spent."""
    import oracle

    t0 = time.perf_counter()
    n = 0
    for D1, D2 in maps[:max_pairs]:
        oracle.frm(D1, D2, 8, 10)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return n, dt, oracle.max_threads()


def run_reference(args):
    """The oracle as the reference arm: same metric, host cores, bounded steps."""
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    from reciprocal_nearest_neighbour_b200 import synth
    import oracle

    w = synth.WORKLOADS[WORKLOAD]
    npairs = max(1, min(args.pairs, args.warmup + args.steps))
    A, B = synth.make_workload_storage(w, "f16", pairs=range(npairs),
                                       workers=min(npairs, os.cpu_count() or 1))
    for s in range(args.warmup):
        oracle.frm(A[s % npairs], B[s % npairs], w.seed_stride, w.max_iter)
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle.frm(A[s % npairs], B[s % npairs], w.seed_stride, w.max_iter)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "pairs/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "pairs_per_step": 1, "H": w.H, "W": w.W, "d": w.d,
                   "seed_stride": w.seed_stride, "max_iter": w.max_iter,
                   "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"one 512x384 pair per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _event_ms(evs_a, evs_b, n):
    return [evs_a[i].elapsed_time(evs_b[i]) for i in range(n)]


def run_native(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import reciprocal_nearest_neighbour_b200 as rnn
    from reciprocal_nearest_neighbour_b200 import _lib, replicas, synth

    world, rank, local = _dist()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        replicas.barrier(world)

    def max_over_ranks(x: float) -> float:
        return replicas.max_over_ranks(x, world, dev)

    lib = _lib.load()
    peaks = _peaks()
    w = synth.WORKLOADS[WORKLOAD]
    P = args.pairs
    pair_ids = replicas.pair_ids(rank, P)         # each rank matches its own pairs
    A_h, B_h = synth.make_workload_storage(w, "f16", pairs=pair_ids,
                                           workers=min(P, max(1, (os.cpu_count() or 2) // world)))
    A_h, B_h = A_h.pin_memory(), B_h.pin_memory()
    A = A_h.to(dev)
    B = B_h.to(dev)
    plan = rnn.FRMPlan(P, w.H, w.W, w.H, w.W, w.d, torch.float16, w.seed_stride, w.max_iter,
                       dev, with_seed_state=True)
    n_per_call_nn = 2 * w.max_iter

    for _ in range(args.warmup):
        plan.run(A, B)
    torch.cuda.synchronize()

    # ---------------------------------------------------------- timed region
    cap = n_per_call_nn * min(args.steps, 20)
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
    for e in ev_a + ev_b:
        e.record()
    torch.cuda.synchronize()
    import ctypes

    h_a = (ctypes.c_void_p * cap)(*[e.cuda_event for e in ev_a])
    h_b = (ctypes.c_void_p * cap)(*[e.cuda_event for e in ev_b])
    rec = ctypes.c_int(0)
    t0e = torch.cuda.Event(enable_timing=True)
    t1e = torch.cuda.Event(enable_timing=True)
    t2e = torch.cuda.Event(enable_timing=True)
    t3e = torch.cuda.Event(enable_timing=True)
    inst_steps = min(args.steps, 20)
    with ClockSampler(dev) as clk:
        barrier()
        torch.cuda.synchronize()
        launches0 = lib.rnn_launch_count()
        t0e.record()
        for _ in range(args.steps):
            plan.run(A, B)
        t1e.record()
        torch.cuda.synchronize()
        launches = lib.rnn_launch_count() - launches0
        barrier()
        # The same steps again with the library's kernel timer on: CUDA events
        # on the launching stream around every fused-kernel launch give its
        # duration.  Those events sit between the launches and keep each kernel
        # from starting under the previous one's tail (programmatic dependent
        # launch), so this pass runs slower and `value` is not taken from it.
        lib.rnn_set_kernel_timer(h_a, h_b, cap, ctypes.byref(rec))
        t2e.record()
        for _ in range(inst_steps):
            plan.run(A, B)
        t3e.record()
        torch.cuda.synchronize()
        lib.rnn_set_kernel_timer(None, None, 0, None)
        barrier()
    clocks = clk.summary()
    step_ms = t0e.elapsed_time(t1e) / args.steps
    step_ms = max_over_ranks(step_ms)
    value = replicas.aggregate_rate(P, world, step_ms)
    rnn.workspace_status(plan.workspace)

    # roofline of the fused similarity+argmax kernel over the recorded launches
    nrec = min(rec.value, cap)
    nn_ms = _event_ms(ev_a, ev_b, nrec)
    seed_state = plan.result.seed_state.cpu().numpy()
    queries_per_call = int(seed_state[:, :, 2].sum())          # sum of active seeds per half-step
    calls_recorded = nrec / n_per_call_nn
    n_cand = w.H * w.W
    flops = 2.0 * w.d * n_cand * queries_per_call * calls_recorded
    nn_time_s = sum(nn_ms) * 1e-3
    achieved_tf = flops / nn_time_s / 1e12
    # the fused kernel is timed inside a region of a few tens of milliseconds,
    # not a seconds-long loop under the power cap: the burst bf16 figure applies
    peak_tf = peaks["bf16_tflops"]
    traffic = (TRAFFIC["frm_nn_bytes_per_launch"]
               if _kernel_sources_sha256() == TRAFFIC["sources_sha256"] else None)
    roofline = {"bound": "tensor", "achieved": round(achieved_tf, 2), "peak": peak_tf,
                "unit": "TFLOP/s", "frac": round(achieved_tf / peak_tf, 4), "traffic": traffic,
                "kernel": "nn_argmax_kernel", "launches": nrec,
                "avg_launch_us": round(1e3 * sum(nn_ms) / max(nrec, 1), 3),
                "flops_per_launch": round(flops / max(nrec, 1), -6),
                "instrumented_ms_per_step": round(t2e.elapsed_time(t3e) / inst_steps, 4),
                "peak_source": f"bf16 burst, {peaks['source']}",
                "active_queries_per_pair": queries_per_call / P}

    # ------------------------------------ the same step as a recorded graph plan
    # Iterations after the last active seed converged launch nothing there; the
    # kernels are the same, so the roofline above stands for both.
    graph_plan = None
    if not args.skip_graph_plan:
        gplan = rnn.FRMGraph(A, B, seed_stride=w.seed_stride, max_iter=w.max_iter,
                             with_seed_state=True)
        for _ in range(args.warmup):
            gplan.launch()
        torch.cuda.synchronize()
        barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(args.steps):
            gplan.launch()
        g1.record()
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps)
        barrier()
        same = bool(torch.equal(gplan.result.count, plan.result.count) and
                    torch.equal(gplan.result.seed_state, plan.result.seed_state))
        # iteration it + 1 runs when some seed makes query 2 it + 1; an iteration is
        # 4 launches (two fused NN launches, two steps)
        max_q = int(seed_state[:, :, 2].max())
        iters_run = 1 + min(w.max_iter - 1, max(0, (max_q - 1) // 2))
        graph_plan = {"value": replicas.aggregate_rate(P, world, graph_ms), "unit": "pairs/s",
                      "ms_per_step": graph_ms, "iterations_run": iters_run,
                      "gpu_launches": int(launches) - 4 * (w.max_iter - iters_run) * args.steps,
                      "results_identical": same}
        gplan.close()

    # ------------------------------------------------------ end to end (host)
    # Every step copies its pairs from pinned host memory and reads its pairs
    # and counts back.  Two input buffers and a copy stream let the copy of
    # step i+1 run while step i matches (the PCIe copy is the longer part).
    pairs_h = [torch.empty_like(plan.result.pairs, device="cpu").pin_memory() for _ in range(2)]
    count_h = [torch.empty_like(plan.result.count, device="cpu").pin_memory() for _ in range(2)]
    bufs = [(A, B), (torch.empty_like(A), torch.empty_like(B))]
    copy_s = torch.cuda.Stream(dev)
    comp_s = torch.cuda.current_stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    for e in freed:
        e.record(comp_s)

    def e2e_step(i):
        a, b = bufs[i % 2]
        with torch.cuda.stream(copy_s):
            copy_s.wait_event(freed[i % 2])          # the buffer's last step has matched
            a.copy_(A_h, non_blocking=True)
            b.copy_(B_h, non_blocking=True)
            copied[i % 2].record(copy_s)
        comp_s.wait_event(copied[i % 2])
        r = plan.run(a, b)
        freed[i % 2].record(comp_s)
        pairs_h[i % 2].copy_(r.pairs, non_blocking=True)
        count_h[i % 2].copy_(r.count, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 20))
    e0.record(comp_s)
    copy_s.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    comp_s.wait_stream(copy_s)
    e1.record(comp_s)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    barrier()
    pairs_h, count_h = pairs_h[0], count_h[0]
    e2e = {"value": round(world * P / (e2e_ms * 1e-3), 2), "unit": "pairs/s",
           "h2d_bytes_per_step": int(A_h.numel() * 2 + B_h.numel() * 2),
           "d2h_bytes_per_step": int(pairs_h.numel() * 4 + count_h.numel() * 4),
           "ms_per_step": round(e2e_ms, 4)}

    # --------------------------------------- exhaustive reciprocal set (rank 0 shape)
    mnn = None
    if not args.skip_mnn:
        mnn = {}
        props = torch.cuda.get_device_properties(dev)
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        peak_cmp = props.multi_processor_count * 128 * peaks["sm_max_mhz"] * 1e6
        for mode, wl, metric in (("quantised", "mnn_512x384_q", "dot"),
                                 ("fp16", "mnn_512x384_f", "dot"),
                                 ("fp16_euclidean", "mnn_512x384_f", "l2")):
            ww = synth.WORKLOADS[wl]
            a, b = synth.make_workload_storage(ww, "f16", pairs=[0])
            a, b = a[0].to(dev), b[0].to(dev)
            out = rnn.mnn_exhaustive(a, b, metric=metric)
            ws = torch.empty(lib.rnn_mnn_workspace_size_ex(ww.H, ww.W, ww.H, ww.W, ww.d,
                                                           _lib.METRICS[metric]),
                             dtype=torch.uint8, device=dev)
            n1 = ww.H * ww.W
            scores = float(n1) * n1
            compares = 2.0 * scores                      # both directions
            rec = {}
            for l2state in ("cold", "warm"):
                reps = args.mnn_reps
                ka = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
                kb = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
                ca = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
                cb = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
                for e in ka + kb:
                    e.record()
                torch.cuda.synchronize()
                ha = (ctypes.c_void_p * reps)(*[e.cuda_event for e in ka])
                hb = (ctypes.c_void_p * reps)(*[e.cuda_event for e in kb])
                r2 = ctypes.c_int(0)
                for _ in range(3):
                    rnn.mnn_exhaustive(a, b, workspace=ws, out=out, metric=metric)
                # the calls, then the same calls with the kernel timer's events
                # around the fused kernel
                for i in range(reps):
                    if l2state == "cold":
                        flush.fill_(i & 0xFF)           # evict the maps from L2
                    ca[i].record()
                    rnn.mnn_exhaustive(a, b, workspace=ws, out=out, metric=metric)
                    cb[i].record()
                torch.cuda.synchronize()
                call_ms = statistics.median(_event_ms(ca, cb, reps))
                lib.rnn_set_kernel_timer(ha, hb, reps, ctypes.byref(r2))
                for i in range(reps):
                    if l2state == "cold":
                        flush.fill_(i & 0xFF)
                    ca[i].record()
                    rnn.mnn_exhaustive(a, b, workspace=ws, out=out, metric=metric)
                    cb[i].record()
                torch.cuda.synchronize()
                lib.rnn_set_kernel_timer(None, None, 0, None)
                inst_ms = statistics.median(_event_ms(ca, cb, reps))
                kern_ms = statistics.median(_event_ms(ka, kb, min(r2.value, reps)))
                rec[l2state] = (call_ms, kern_ms, inst_ms)
            call_ms, kern_ms, inst_ms = rec["cold"]
            achieved_cmp = compares / (kern_ms * 1e-3)
            mnn[mode] = {
                "value": round(scores / (call_ms * 1e-3), -6), "ms_per_call": round(call_ms, 4),
                "kernel_ms": round(kern_ms, 4), "instrumented_ms_per_call": round(inst_ms, 4),
                "warm": {"ms_per_call": round(rec["warm"][0], 4),
                         "kernel_ms": round(rec["warm"][1], 4)},
                "pairs": int(out.count.item()),
                "roofline": {"bound": "alu", "achieved": round(achieved_cmp / 1e12, 3),
                             "peak": round(peak_cmp / 1e12, 3), "unit": "Tcompare/s",
                             "frac": round(achieved_cmp / peak_cmp, 4),
                             "frac_call": round(compares / (call_ms * 1e-3) / peak_cmp, 4)}}
        mnn["unit"] = "pair-scores/s"
        mnn["note"] = ("512x384 d=24; cold = 256 MB L2 flush before each call; frac: 2*N1*N2 "
                       "compares over the fused kernel time vs SMs x 128 x max MHz; kernel_ms "
                       "from a second pass with timing events around the kernel "
                       "(instrumented_ms_per_call)")
        del flush

    # ------------- one pair per call (the single-pair entry point), 512x384
    single = None
    if not args.skip_mnn:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        a1, b1 = A[0].contiguous(), B[0].contiguous()
        ws1 = torch.empty(lib.rnn_frm_workspace_size(1, w.H, w.W, w.H, w.W, w.d, w.seed_stride),
                          dtype=torch.uint8, device=dev)

        def one():
            return rnn.frm_match(a1, b1, w.seed_stride, w.max_iter, workspace=ws1)

        for _ in range(3):
            one()
        cold_ms, r1 = _timed_calls(one, 20, flush)
        warm_ms, _ = _timed_calls(one, 20, None)
        single = {"value": round(1e3 / cold_ms, 1), "unit": "pairs/s",
                  "ms_per_call": round(cold_ms, 4),
                  "warm": {"value": round(1e3 / warm_ms, 1), "ms_per_call": round(warm_ms, 4)},
                  "pairs_out": int(r1.count.sum().item()),
                  "note": "rnn_frm_match, one pair per call; cold = L2 flushed"}
        del flush

    # ------ one exhaustive set split over the ranks (row slices + all-gather)
    sharded = None
    if world > 1 and not args.skip_mnn:
        ww = synth.WORKLOADS["mnn_512x384_q"]
        a, b = synth.make_workload_storage(ww, "f16", pairs=[0])
        a, b = a[0].to(dev), b[0].to(dev)
        for _ in range(3):
            replicas.mnn_sharded(a, b, world, rank)
        torch.cuda.synchronize()
        barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        reps = 5
        s0.record()
        for _ in range(reps):
            pr, cnt = replicas.mnn_sharded(a, b, world, rank)
        s1.record()
        torch.cuda.synchronize()
        own_ms = s0.elapsed_time(s1) / reps
        sh_ms = max_over_ranks(own_ms)
        barrier()
        n1 = ww.H * ww.W
        sharded = {"value": round(float(n1) * n1 / (sh_ms * 1e-3), -6),
                   "unit": "pair-scores/s", "ms_per_call": round(sh_ms, 4),
                   "rank0_ms": round(own_ms, 4),
                   "per_rank_value": round(float(n1) * n1 / world / (sh_ms * 1e-3), -6),
                   "pairs": int(cnt.item()),
                   "note": f"one 512x384 set over {world} ranks: row-slice NN, all-gather of "
                           "the argmax arrays, mutual test"}

    # ---------------- FRM options on the step's pairs: given starts, basin mode
    options = None
    if not args.skip_mnn:
        options = {}
        # starts one pixel right of and below each grid seed (3072 a pair)
        seeds = torch.arange(w.H * w.W, device=dev, dtype=torch.int32).reshape(w.H, w.W)
        off = w.seed_stride // 2 + 1
        starts = seeds[off::w.seed_stride, off::w.seed_stride].reshape(1, -1).repeat(P, 1)
        cases = (("refine", dict(max_iter=1, init=starts, pixel_tol=1.5), starts.shape[1] * P,
                  "refined starts/s (one round trip, pixel_tol 1.5)"),
                 ("basin", dict(seed_stride=w.seed_stride, max_iter=w.max_iter, with_basin=True),
                  P, "FRM pairs/s with the basin output"))
        for name, kw, units, what in cases:
            for _ in range(2):
                r = rnn.frm_match_ex(A, B, **kw)
            reps = 10
            oa = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
            ob = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
            for i in range(reps):
                oa[i].record()
                r = rnn.frm_match_ex(A, B, **kw)
                ob[i].record()
            torch.cuda.synchronize()
            ms = statistics.median(_event_ms(oa, ob, reps))
            options[name] = {"metric": what, "value": units / (ms * 1e-3),
                             "unit": "starts/s" if name == "refine" else "pairs/s",
                             "ms_per_call": ms, "pairs_per_call": P,
                             "outputs": int(r.count.sum().item()),
                             "note": "includes the binding's output and workspace allocation"}

    # ------------------------- 3-D point maps (the K-d tree workload, exact NN)
    pts = None if args.skip_mnn else _points_leg(dev, lib, w, P, 10)
    # ------------- coarse-to-fine: 1024x768, d = 32, coarse 80x64 cells, d = 256
    c2f = None if args.skip_mnn else _c2f_leg(dev, lib, 10)
    # -------------- the other FRM configurations: 64 pairs of 512x288; 1024x768
    configs = None
    if not args.skip_mnn:
        configs = {n: _frm_config_leg(dev, n, 5) for n in ("frm_batched_64x512x288",
                                                          "frm_1024x768")}

    # ----------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        maps = [(A_h[i], B_h[i]) for i in range(min(P, 4))]
        n, dt, cores = _oracle_frm_pairs_per_s(maps, args.cpu_budget_s, 4)
        cpu = {"value": round(n / dt, 4), "unit": "pairs/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} of this step's 512x384 pairs, whole FRM loop, f64"}

    if rank == 0:
        # the secondary legs first, on a line of their own, so that the final
        # line (the headline numbers) stays short
        print(json.dumps({"bench_legs": {"frm_options": options, "frm_graph_plan": graph_plan,
                                         "points": pts, "coarse_to_fine": c2f,
                                         "frm_configs": configs}}), flush=True)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "pairs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "pairs_per_step": P, "H": w.H, "W": w.W,
                       "d": w.d, "seed_stride": w.seed_stride, "max_iter": w.max_iter,
                       "global_batch": world * P, "parallelism": f"replicas x{world}",
                       "l2": f"step inputs {2 * A_h.numel() * 2 / 1e6:.0f} MB > 126 MB L2"},
            "e2e": e2e, "roofline": roofline, "mnn": mnn, "frm_single_pair": single,
            "mnn_sharded": sharded, "cpu_baseline": cpu,
            "clocks": clocks, "gpu_launches": int(launches),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def _timed_calls(fn, reps, flush):
    """Median CUDA-event time of `reps` calls, each after an L2 flush (none
    when `flush` is None)."""
    import torch
    oa = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    ob = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    r = None
    for i in range(reps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        oa[i].record()
        r = fn()
        ob[i].record()
    torch.cuda.synchronize()
    return statistics.median(_event_ms(oa, ob, reps)), r


def _points_leg(dev, lib, w, P, reps, warmup=3):
    """Reciprocal set and FRM on 512x384 point maps (fp32, exact Euclidean NN)."""
    import numpy as np
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    from reciprocal_nearest_neighbour_b200 import synth
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    pm = [synth.pointmap_pair(700 + i, w.H, w.W) for i in range(P)]
    p1 = torch.from_numpy(np.stack([m[0] for m in pm]).astype(np.float32)).to(dev)
    p2 = torch.from_numpy(np.stack([m[1] for m in pm]).astype(np.float32)).to(dev)
    n1 = w.H * w.W
    ws_m = torch.empty(lib.rnn_pts_mnn_workspace_size(w.H, w.W, w.H, w.W),
                       dtype=torch.uint8, device=dev)
    ws_f = torch.empty(lib.rnn_pts_frm_workspace_size(P, w.H, w.W, w.H, w.W, w.seed_stride, -1),
                       dtype=torch.uint8, device=dev)
    cases = (("mnn", lambda: rnn.pts_mnn(p1[0], p2[0], workspace=ws_m), 2 * n1, "queries/s",
              "exhaustive reciprocal set of two 512x384 point maps (both directions)"),
             ("frm", lambda: rnn.pts_frm_match(p1, p2, seed_stride=w.seed_stride,
                                               max_iter=w.max_iter, workspace=ws_f),
              P, "pairs/s", f"FRM on {P} pairs of 512x384 point maps, stride "
              f"{w.seed_stride}, max_iter {w.max_iter}"))
    out = {}
    for name, fn, units, unit, what in cases:
        for _ in range(warmup):
            fn()
        ms, r = _timed_calls(fn, reps, flush)
        out[name] = {"metric": what, "value": units / (ms * 1e-3), "unit": unit,
                     "ms_per_call": ms, "outputs": int(r.count.sum().item()), "dtype": "f32",
                     "note": "includes the binding's output allocation; 256 MB L2 flush "
                             "before every call"}
    return out


def _graph_of(fn):
    """fn() recorded into a torch CUDA graph (one eager call on a side stream
    first); FRM calls inside it record their later iterations as conditional
    nodes.  Returns the graph and the outputs its replays rewrite."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    torch.cuda.synchronize()
    return g, out


def _graph_timing(fn, ref_count, reps, flush):
    """Median time of replays of fn() recorded as a graph, and whether a
    replay's counts equal `ref_count` (a copy of the eager call's)."""
    import torch
    g, out = _graph_of(fn)
    ms, _ = _timed_calls(lambda: (g.replay(), out)[1], reps, flush)
    same = bool(torch.equal(out.count, ref_count))
    del g
    return ms, same


def _c2f_leg(dev, lib, reps, warmup=3):
    """Coarse-to-fine: 1024x768 maps (d = 32), coarse M on 80x64 cells (d = 256)."""
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    from reciprocal_nearest_neighbour_b200 import synth
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    big = synth.WORKLOADS["frm_1024x768"]
    F1, F2 = synth.make_workload(big)
    C1 = synth.coarse_map(F1, 64, 80, dc=256, seed=11)
    C2 = synth.coarse_map(F2, 64, 80, dc=256, seed=11)
    c1, c2, f1, f2 = (synth.to_storage(x, "f16").to(dev) for x in (C1, C2, F1, F2))
    kw = dict(crop=(384, 512), seed_stride=big.seed_stride, max_iter=big.max_iter)
    ws_c = torch.empty(lib.rnn_c2f_workspace_size(64, 80, 64, 80, 256, big.H, big.W, big.H,
                                                  big.W, big.d, 0, 384, 512, big.seed_stride),
                       dtype=torch.uint8, device=dev)

    def fn():
        return rnn.c2f_match(c1, c2, f1, f2, workspace=ws_c, **kw)

    for _ in range(warmup):
        fn()
    ms, r = _timed_calls(fn, reps, flush)
    gms, same = _graph_timing(fn, r.count.clone(), reps, flush)
    return {"metric": "coarse-to-fine image pairs/s: 1024x768 maps, d=32, coarse M on 80x64 "
                      "cells (d=256), 2x2 crops of 512x384, FRM stride 8, max_iter 15",
            "value": 1e3 / ms, "unit": "pairs/s", "ms_per_call": ms,
            "graph": {"value": 1e3 / gms, "ms_per_call": gms, "counts_identical": same,
                      "note": "the call recorded into a CUDA graph and replayed: FRM "
                              "iterations after convergence launch nothing"},
            "outputs": int(r.count.item()), "crops_on": int(r.crops[:, 5].sum().item()),
            "dtype": "f16",
            "note": "includes the binding's output allocation; 256 MB L2 flush before every call"}


def _frm_config_leg(dev, name, reps, warmup=3):
    """FRM on a whole workload (all its pairs in one batched call): pairs/s,
    and the tensor work it did (2*d*N*sum of live queries) per second."""
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    from reciprocal_nearest_neighbour_b200 import synth
    w = synth.WORKLOADS[name]
    A_h, B_h = synth.make_workload_storage(w, "f16", workers=min(w.pairs, os.cpu_count() or 1))
    A, B = A_h.to(dev), B_h.to(dev)
    plan = rnn.FRMPlan(w.pairs, w.H, w.W, w.H, w.W, w.d, torch.float16, w.seed_stride,
                       w.max_iter, dev, with_seed_state=True)
    for _ in range(warmup):
        plan.run(A, B)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ms, r = _timed_calls(lambda: plan.run(A, B), reps, flush)
    queries = int(r.seed_state[:, :, 2].sum().item())
    flops = 2.0 * w.d * w.H * w.W * queries
    gms, same = _graph_timing(lambda: plan.run(A, B), r.count.clone(), reps, flush)
    return {"metric": f"FRM image pairs/s, {w.pairs} pair(s) of {w.W}x{w.H}, d={w.d}, stride "
                      f"{w.seed_stride}, max_iter {w.max_iter}",
            "value": w.pairs / (ms * 1e-3), "unit": "pairs/s", "ms_per_call": ms,
            "outputs": int(r.count.sum().item()), "active_queries_per_pair": queries / w.pairs,
            "tensor_tflops_per_call": flops / (ms * 1e-3) / 1e12, "dtype": "f16",
            "graph": {"value": w.pairs / (gms * 1e-3), "ms_per_call": gms,
                      "counts_identical": same,
                      "note": "the call recorded into a CUDA graph and replayed: iterations "
                              "after convergence launch nothing"},
            "note": "whole-call time (256 MB L2 flush before every call); the tensor rate counts "
                    "the live queries' flops over the call, not one kernel"}


def run_leg(name, steps, warmup):
    """One leg alone (for profiling): its calls, then one JSON line."""
    import torch
    from reciprocal_nearest_neighbour_b200 import _lib, synth
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name == "points":
        res = _points_leg(dev, lib, synth.WORKLOADS[WORKLOAD], 8, steps, warmup)
    elif name == "c2f":
        res = _c2f_leg(dev, lib, steps, warmup)
    else:
        res = _frm_config_leg(dev, name, steps, warmup)
    print(json.dumps({"leg": name, "result": res}), flush=True)
    return 0


def run_nn_case(nq, d, nx):
    """One small nearest-neighbour case for an ncu capture of the fused kernel."""
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    gen = torch.Generator(device="cuda").manual_seed(0)
    Q = torch.randn(nq, d, device="cuda", generator=gen).half()
    X = torch.randn(nx, d, device="cuda", generator=gen).half()
    for _ in range(3):
        idx, sc = rnn.nn_argmax(Q, X)
    torch.cuda.synchronize()
    print(f"nn-case {nq}x{nx} d={d}: idx[0]={int(idx[0])} score[0]={float(sc[0]):.6f}")
    return 0


def run_mnn_case(mode):
    """The exhaustive set at 512x384, d=24 three times (for an ncu capture of
    the one-pass kernel): mode "q" quantised maps, "f" unit-norm fp16 maps."""
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    from reciprocal_nearest_neighbour_b200 import synth
    w = synth.WORKLOADS["mnn_512x384_q" if mode == "q" else "mnn_512x384_f"]
    a, b = synth.make_workload_storage(w, "f16", pairs=[0])
    a, b = a[0].cuda(), b[0].cuda()
    for _ in range(3):
        r = rnn.mnn_exhaustive(a, b)
    torch.cuda.synchronize()
    print(f"mnn-case {w.name}: |M| = {int(r.count.item())}")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--pairs", type=int, default=8, help="image pairs per step and rank")
    ap.add_argument("--mnn-reps", type=int, default=10)
    ap.add_argument("--skip-mnn", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--skip-graph-plan", action="store_true",
                    help="do not time the step as a recorded graph plan")
    ap.add_argument("--leg", choices=["points", "c2f", "frm_batched_64x512x288", "frm_1024x768"],
                    help="run one secondary leg alone (for profiling) and exit")
    ap.add_argument("--nn-case", type=int, nargs=3, metavar=("NQ", "D", "NX"),
                    help="profiling aid: run nn_argmax three times on seeded fp16 "
                         "queries/candidates of these sizes and exit (no timing)")
    ap.add_argument("--mnn-case", choices=["q", "f"],
                    help="profiling aid: run the 512x384 exhaustive set three times on the "
                         "quantised (q) or fp16 (f) maps and exit (no timing)")
    args = ap.parse_args(argv)
    if args.mnn_case:
        return run_mnn_case(args.mnn_case)
    if args.leg:
        return run_leg(args.leg, args.steps, args.warmup)
    if args.nn_case:
        return run_nn_case(*args.nn_case)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
