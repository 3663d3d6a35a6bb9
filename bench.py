#!/usr/bin/env python
"""StateKV streaming-prefill benchmark: frames/s per layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 8b_layer] [--l2 flush|resident]

One step = one StateKV cache-builder step (attention, score pass, top-B select,
gather + append) for one layer and one frame, in steady state (the compressed
state is full).  Before the W untimed warm-up steps the stream is run through
ceil(B/T) fill frames.  Inputs are seeded synthetic frames already resident in
device memory.  Each timed step is bracketed by CUDA events on the launching
stream; with --l2 flush (default) a 256 MiB buffer is written between steps,
outside the events.  For N > 1 every rank runs an independent replica stream
(no collective on the data path); value = all frames / max-over-ranks time.

--impl reference times the float64 CPU oracle (rank 0 only) on the same
workload: each step is one oracle step on a sample of the KV heads, scaled to
the whole layer.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_selection_b200 import synthetic as Syn  # noqa: E402

METRIC = "StateKV prefill frames/s per layer (8B shape, B=4096); % tensor-pipe peak"
UNIT = "frames/s per layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers --
def rank_info():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def load_peaks(path=None):
    """Roofline denominators: the measured peaks file when it gives them
    (positive numbers under the fallback's keys), else the fallback figures;
    the second value says which ("measured", "measured+fallback" when the
    file gives only some of them, or "fallback")."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks, found = dict(FALLBACK_PEAKS), 0
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
        except (OSError, ValueError):
            d = {}
        for k in FALLBACK_PEAKS:
            v = d.get(k) if isinstance(d, dict) else None
            if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
                peaks[k] = float(v)
                found += 1
    if found == len(FALLBACK_PEAKS):
        return peaks, "measured"
    return peaks, ("measured+fallback" if found else "fallback")


def step_work(wl, m, S=1, causal=True):
    """Algorithmic work of one step at C length m."""
    T, Hq, Hkv, d = wl.T, wl.Hq, wl.Hkv, wl.d
    esize = 2 if wl.dtype == "bf16" else 4
    pairs = T * m + (T * (T + 1) // 2 if causal else T * T)   # visible (query, key) pairs per head
    qk = 2 * S * Hq * d * pairs
    m_new = min(wl.B, m + T)
    L = m + T
    gather_bytes = S * Hkv * (2 * 2 * m_new * d * esize + 2 * 8 * m_new) \
        + S * Hkv * 2 * 2 * T * d * esize + S * T * 8
    select_bytes = S * Hkv * L * 4 * 2 + S * Hkv * wl.B * 12
    return {"attention": ("tensor", 2 * qk), "score": ("tensor", qk),
            "select": ("hbm", select_bytes), "gather": ("hbm", gather_bytes)}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            # STATEKV_CLOCKS_DIR keeps the raw samples for inspection; by
            # default they go to the system temporary directory
            out_dir = os.environ.get("STATEKV_CLOCKS_DIR") or tempfile.gettempdir()
            self.path = os.path.join(out_dir, f"clocks_rank{self.gpu}_{os.getpid()}.csv")
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_stage, workload):
    """Per-launch DRAM bytes from a committed ncu summary, if it is current."""
    p = os.path.join(ROOT, "profiles", f"traffic_{kernel_stage}_{workload}.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        if d.get("source_sha") != source_hash(d["sources"]):
            return None
        return float(d["dram_bytes_per_launch"])
    except Exception:
        return None


def dist_max(x: float, device) -> float:
    """Max of a per-rank number over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def dist_sum(x: float, device) -> float:
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def replica_throughput(local_frames: int, local_ms: float, device) -> tuple:
    """Whole-job frames/s of independent replicas: all frames over the slowest
    rank's time.  Returns (value, max_ms)."""
    max_ms = dist_max(local_ms, device)
    frames = dist_sum(local_frames, device)
    return frames / (max_ms / 1e3), max_ms


# ------------------------------------------------------------------ our arm --
def make_frames(wl, n_distinct, stream, dev):
    fr = Syn.gen_frames(wl, n_distinct, stream=stream)
    q = torch.stack([f[0] for f in fr]).to(dev)
    k = torch.stack([f[1] for f in fr]).to(dev)
    v = torch.stack([f[2] for f in fr]).to(dev)
    return fr, q, k, v


def run_ours(args, wl):
    from kv_cache_selection_b200 import statekv as SKV

    rank, local_rank, world = rank_info()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    K, W = args.steps, args.warmup
    fill = math.ceil(wl.B / wl.T)
    n_enq = min(K, 50)
    total_frames = fill + W + 3 * K + n_enq   # timed pass, two per-stage profiling passes, host enqueue pass
    n_distinct = min(total_frames, args.distinct_frames)
    fr_cpu, Q, Kf, Vf = make_frames(wl, n_distinct, rank, dev)
    pos_all = torch.arange(total_frames * wl.T, dtype=torch.int32, device=dev).view(total_frames, wl.T)
    out = torch.empty((wl.T, wl.Hq, wl.d), dtype=wl.torch_dtype, device=dev)
    h = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=total_frames, dtype=wl.dtype)
    h.reserve_layers(1)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev) if args.l2 == "flush" else None

    def step(n):
        i = n % n_distinct
        h.prefill_frame(0, Q[i], Kf[i], Vf[i], pos_all[n], out)

    for n in range(fill + W):
        step(n)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    launches0 = h.kernel_launches()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for j in range(K):
        if flush is not None:
            flush.fill_(j)
        ev[j][0].record()
        step(fill + W + j)
        ev[j][1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = h.kernel_launches() - launches0
    clk = clocks.stop()
    # second pass of K steps with the library's per-kernel event pairs (they
    # serialise the kernels, so the headline above is taken without them)
    # Each step is queued behind a ~100 us spin kernel, so that the host has
    # queued the whole step (with its event records) before the GPU reaches
    # it: the event pairs then time the kernels, not the host's launch calls.
    h.profile(True)
    for j in range(K):
        if flush is not None:
            flush.fill_(j)
        torch.cuda._sleep(200_000)
        step(fill + W + K + j)
    torch.cuda.synchronize()
    stages = h.profile_read()
    # third pass: the attention and the merge of its key splits under one
    # event pair, the merge launched right behind the attention (programmatic
    # dependent launch, as the step chains its kernels)
    h.profile(2)
    for j in range(K):
        if flush is not None:
            flush.fill_(j)
        torch.cuda._sleep(200_000)
        step(fill + W + 2 * K + j)
    torch.cuda.synchronize()
    chained = h.profile_read().get("attention_chained", (0.0, 0))
    h.profile(False)
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    value, ms_total = replica_throughput(K, sum(ms_steps), dev)

    # ---- end to end through the host-buffer C-ABI call (pinned host memory):
    # every step copies its frame in and its output back inside the timed
    # region; the K steps are timed as one region (consecutive steps may overlap
    # their copies with the previous step's kernels, as a streaming caller would)
    e2e = None
    if not args.no_e2e:
        he = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=total_frames, dtype=wl.dtype)
        he.reserve_layers(1)
        host_frames = [(f[0].contiguous().pin_memory(), f[1].contiguous().pin_memory(),
                        f[2].contiguous().pin_memory()) for f in fr_cpu]
        host_pos = torch.arange(total_frames * wl.T, dtype=torch.int32).view(total_frames, wl.T).pin_memory()
        host_out = [torch.empty((wl.T, wl.Hq, wl.d), dtype=wl.torch_dtype).pin_memory() for _ in range(2)]

        def host_step(n):
            i = n % n_distinct
            he.prefill_frame_host(0, host_frames[i][0], host_frames[i][1], host_frames[i][2], host_pos[n],
                                  host_out[n & 1])

        for n in range(fill + W):
            host_step(n)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record()
        th0 = time.perf_counter()
        for j in range(K):
            host_step(fill + W + j)
        host_call_us = (time.perf_counter() - th0) / K * 1e6
        e1.record()
        torch.cuda.synchronize()
        e2e_value, e2e_ms = replica_throughput(K, e0.elapsed_time(e1), dev)
        esize = 2 if wl.dtype == "bf16" else 4
        h2d = (wl.T * wl.Hq * wl.d + 2 * wl.T * wl.Hkv * wl.d) * esize + wl.T * 4
        d2h = wl.T * wl.Hq * wl.d * esize
        # the step's copies alone, from and to the same pinned host tensors the
        # end-to-end loop used (one direction at a time, on a side stream): the
        # floor that the end-to-end step is set against
        hq, hk, hv = host_frames[0]
        dq, dk, dv = torch.empty_like(hq, device=dev), torch.empty_like(hk, device=dev), torch.empty_like(hv, device=dev)
        dp = torch.empty_like(host_pos[0], device=dev)
        dout = torch.empty_like(host_out[0], device=dev)
        cs = torch.cuda.Stream()

        def h2d_copy():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dp.copy_(host_pos[0], non_blocking=True)

        def d2h_copy():
            host_out[0].copy_(dout, non_blocking=True)

        link = {}
        for name, fn in (("h2d", h2d_copy), ("d2h", d2h_copy)):
            with torch.cuda.stream(cs):
                for _ in range(3):
                    fn()
                c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                c0.record()
                for _ in range(20):
                    fn()
                c1.record()
            c1.synchronize()
            us = c0.elapsed_time(c1) / 20 * 1e3
            n_b = h2d if name == "h2d" else d2h
            link[name + "_us"] = round(us, 2)
            link[name + "_gbs"] = round(n_b / (us * 1e-6) / 1e9, 2)
        # both directions at once, on two streams
        cs2 = torch.cuda.Stream()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        c0.record()
        cs.wait_event(c0)
        cs2.wait_event(c0)
        for _ in range(20):
            with torch.cuda.stream(cs):
                h2d_copy()
            with torch.cuda.stream(cs2):
                d2h_copy()
        e_a, e_b = torch.cuda.Event(), torch.cuda.Event()
        e_a.record(cs)
        e_b.record(cs2)
        torch.cuda.current_stream().wait_event(e_a)
        torch.cuda.current_stream().wait_event(e_b)
        c1.record()
        c1.synchronize()
        link["both_directions_us"] = round(c0.elapsed_time(c1) / 20 * 1e3, 2)
        e2e = {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 5),
               "path": "statekv_prefill_frame_host (pinned host buffers; the library stages the copies)",
               "l2": "not flushed (host copies dominate)",
               "host_us_per_call": round(host_call_us, 2),
               "pcie_copies_alone": link}
        he.close()

    # ---- host enqueue cost of one step (back-to-back calls, no synchronisation)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for j in range(n_enq):
        step(fill + W + 3 * K + j)
    host_enqueue_us = (time.perf_counter() - t0) / n_enq * 1e6
    torch.cuda.synchronize()

    # ---- flatness: the full 512-frame stream of the 8B layer, per-frame time
    flat = dec = cross = None
    if not args.no_flatness and wl.name == "8b_layer":
        flat, dec = flatness_report(SKV, wl, dev)
        cs = ClockSampler(local_rank)
        cs.start()
        cross = sweep_report([32, 64, 128, 256], [4096], dev)
        cross["clocks"] = cs.stop()

    if rank != 0:
        h.close()
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    work = step_work(wl, wl.B)
    # the merge of the attention's key splits is part of (a): charge it there.
    # (a)'s time is the third pass's event pair around the attention and its
    # merge, chained as in the step; the kernel's own event time and the merge
    # launched on its own (second pass) are reported beside it.
    attn_kernel_us = merge_alone_us = None
    if stages.get("attention", (0, 0))[1]:
        attn_kernel_us = stages["attention"][0] / stages["attention"][1] * 1e3
    if stages.get("attention_combine", (0, 0))[1]:
        merge_alone_us = stages["attention_combine"][0] / stages["attention_combine"][1] * 1e3
        if not chained[1]:
            a_ms, a_n = stages["attention"]
            stages["attention"] = (a_ms + stages["attention_combine"][0], a_n)
    stages.pop("attention_combine", None)
    if chained[1]:
        stages["attention"] = chained
    stage_us = {k: (v[0] / max(v[1], 1)) * 1e3 for k, v in stages.items() if v[1]}
    dominant = max(stage_us, key=lambda k: stages[k][0])
    bound, amount = work.get(dominant, ("tensor", 0))
    avg_s = stage_us[dominant] / 1e6
    if bound == "tensor":
        achieved = amount / avg_s / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = amount / avg_s / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    roofline = {"kernel": dominant, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
                "unit": unit, "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} ({'bf16 burst' if bound == 'tensor' else 'copy'})",
                "algorithmic_per_launch": amount,
                "traffic": ncu_traffic(dominant, wl.name)}
    if dominant == "attention" and attn_kernel_us and bound == "tensor":
        roofline["kernel_alone"] = {"us": round(attn_kernel_us, 2),
                                    "achieved": round(amount / (attn_kernel_us / 1e6) / 1e12, 2),
                                    "frac": round(amount / (attn_kernel_us / 1e6) / 1e12 / peak, 4),
                                    "note": "the attention kernel's own event time, without its split merge"}
        if merge_alone_us is not None:
            roofline["merge_launched_alone_us"] = round(merge_alone_us, 2)
    per_stage = {}
    for k, us in stage_us.items():
        b, amt = work.get(k, ("", 0))
        if b == "tensor":
            per_stage[k] = {"us": round(us, 2), "tflops": round(amt / us / 1e6, 1),
                            "frac": round(amt / us / 1e6 / peaks["bf16_tflops"], 4)}
        elif b == "hbm":
            per_stage[k] = {"us": round(us, 2), "gbs": round(amt / us / 1e3, 1),
                            "frac": round(amt / us / 1e3 / peaks["hbm_gbs"], 4)}
        else:
            per_stage[k] = {"us": round(us, 2)}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, h, fr_cpu, total_frames, n_distinct, budget_s=args.cpu_budget)
    h.close()

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms_total / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: Hq={wl.Hq} Hkv={wl.Hkv} d={wl.d} T={wl.T} B={wl.B}, "
                               f"steady state (C full), frame-causal, global select",
                   "global_batch": world, "seq_len": wl.T, "frames_per_rank": total_frames,
                   "l2": ("256 MiB buffer written between timed steps (outside the events)"
                          if args.l2 == "flush" else "not flushed (C stays L2-resident across frames)"),
                   "parallelism": f"replicas x{world} (no data-path collective)"},
        "roofline": roofline,
        "stages_us": per_stage,
        "stages_note": ("per-kernel CUDA events in a second pass of K steps (events serialise the kernels; "
                        "each step queued behind a spin kernel so the host's launch calls are not timed); "
                        "attention: one event pair around the attention kernel and the merge of its key "
                        "splits, launched right behind it (programmatic dependent launch), in a third pass "
                        "of K steps"),
        "step_us_p50": round(statistics.median(ms_steps) * 1e3, 2),
        "step_us_p99": round(sorted(ms_steps)[int(0.99 * (len(ms_steps) - 1))] * 1e3, 2),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
        "gpu_launches_per_step": launches / K, "host_enqueue_us_per_step": round(host_enqueue_us, 2),
        "clocks": clk, "flatness": flat, "decode": dec, "crossover": cross,
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, h, fr_cpu, n_next, n_distinct, budget_s=20.0, kv_heads=None):
    """The oracle, as it stands, on a bounded sample of the same workload: steady
    state steps from the GPU's own compressed state, on a subset of the KV heads
    (each with its G query heads), scaled to the whole layer."""
    from threadpoolctl import threadpool_info
    from oracle import statekv_oracle as O

    C = h.get_compressed(0)
    m = C["len"]
    G = wl.Hq // wl.Hkv
    kvh = kv_heads or 1
    st = O.LayerState.from_compressed(C["k"][0, :kvh, :m].cpu(), C["v"][0, :kvh, :m].cpu(),
                                      C["pos"][0, :kvh, :m].cpu().numpy())
    frames_done = 0
    t0 = time.perf_counter()
    n = n_next
    while True:
        q, k, v, _ = fr_cpu[n % n_distinct]
        pos = torch.arange(n * wl.T, (n + 1) * wl.T).numpy()
        st, _ = O.statekv_step(st, q[:, :kvh * G], k[:, :kvh], v[:, :kvh], pos, wl.B)
        frames_done += 1
        n += 1
        el = time.perf_counter() - t0
        if el > budget_s or frames_done >= 64:
            break
    threads = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
    frac = kvh / wl.Hkv
    value = frames_done * frac / el
    # the same oracle restricted to one BLAS thread, on a few more frames
    from threadpoolctl import threadpool_limits
    one_frames, t1 = 0, time.perf_counter()
    with threadpool_limits(limits=1):
        while True:
            q, k, v, _ = fr_cpu[n % n_distinct]
            pos = torch.arange(n * wl.T, (n + 1) * wl.T).numpy()
            st, _ = O.statekv_step(st, q[:, :kvh * G], k[:, :kvh], v[:, :kvh], pos, wl.B)
            one_frames += 1
            n += 1
            el1 = time.perf_counter() - t1
            if el1 > budget_s / 4 or one_frames >= 8:
                break
    return {"value": round(value, 5), "unit": UNIT, "cores": int(max(threads) if threads else 1),
            "host_cpus": os.cpu_count(), "kind": "oracle",
            "value_1_core": round(one_frames * frac / el1, 5),
            "sample": f"{frames_done} steady-state frames of {wl.name} on {kvh} of {wl.Hkv} KV heads "
                      f"({kvh * G} query heads), float64 numpy oracle, {el:.1f} s; value scaled by "
                      f"{wl.Hkv}/{kvh}; value_1_core: {one_frames} further frames with one BLAS thread, "
                      f"{el1:.1f} s"}


# ------------------------------------------------------------ report modes --
def _flush_l2(buf, j):
    if buf is not None:
        buf.fill_(j)


def _per_frame_times(step_fn, n_frames, flush, dev):
    """Device time of each step (CUDA events, L2 flushed between steps)."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_frames)]
    torch.cuda.synchronize()
    for n in range(n_frames):
        _flush_l2(flush, n)
        ev[n][0].record()
        step_fn(n)
        ev[n][1].record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) * 1e3 for a, b in ev]  # us


def _flatness(us, first):
    import numpy as np
    y = np.asarray(us[first:])
    x = np.arange(first, len(us))
    slope = float(np.polyfit(x, y, 1)[0]) if len(y) > 2 else 0.0
    p50 = float(np.percentile(y, 50))
    p99 = float(np.percentile(y, 99))
    return {"from_frame": first, "mean_us": round(float(y.mean()), 2), "p50_us": round(p50, 2),
            "p99_us": round(p99, 2), "p99_over_p50": round(p99 / p50, 3),
            "slope_us_per_frame": round(slope, 5),
            "slope_over_512_frames_pct": round(100 * slope * 512 / p50, 2)}


def flatness_report(SKV, wl, dev):
    """The whole 512-frame stream of the 8B-class layer from an empty state:
    device time of every frame (CUDA events, L2 flushed between frames), the
    least-squares slope over the steady state and its p99/p50, with the SM
    clocks sampled while it runs."""
    wl = Syn.workload("8b_layer")
    q, k, v, pos = Syn.gen_frames_device(wl, wl.frames, device=dev)
    h = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype=wl.dtype)
    h.reserve_layers(1)
    out = torch.empty_like(q[0])
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    us = _per_frame_times(lambda n: h.prefill_frame(0, q[n], k[n], v[n], pos[n], out), wl.frames, flush, dev)
    clk = clocks.stop()
    fill = math.ceil(wl.B / wl.T)
    rep = {"workload": "8b_layer: 512 frames from an empty state, B=4096, device-drawn synthetic frames",
           "l2": "flushed between frames", "fill_frames": fill,
           "fill_us": [round(x, 1) for x in us[:fill]], "steady": _flatness(us, fill),
           "per_frame_us_every_32": [round(x, 1) for x in us[::32]], "clocks": clk}
    del q, k, v, pos
    dec = decode_report(h, wl, dev, flush)
    h.close()
    return rep, dec


def decode_report(h, wl, dev, flush, n_texts=(1, 16, 64), reps=20):
    """Decode attention of n text tokens over the layer's whole detailed state
    (512 frames = 131,072 tokens): device time per call (CUDA events, L2
    flushed before each call) against its roofline.  The algorithmic bytes
    are D's K and V read once (2 * Hkv * N * d * 2) plus the text q, k, v, out;
    the algorithmic FLOPs are 4 * Hq * d * (n * N + n (n + 1) / 2) (QK^T and
    PV over D and the causal text block).  The bound is whichever of the two
    takes longer at the peaks: HBM for a few text tokens, the tensor pipe once
    G * n query rows share each K/V row (n = 64 at G = 7)."""
    peaks, src = load_peaks()
    N = h.frames(0) * wl.T
    res = {"workload": f"8b_layer: decode over D after {h.frames(0)} frames ({N} tokens)", "per_n_text": {}}
    for n in n_texts:
        wl_t = Syn.workload(wl.name, T=n, dist="iid", n_sinks=0, drift=0)
        q, k, v, _ = Syn.gen_frames_device(wl_t, 1, device=dev)
        q, k, v = q[0], k[0], v[0]
        out = torch.empty_like(q)
        h.decode(0, q, k, v, out=out, with_lse=False)   # warm-up (allocates split scratch)
        ts = []
        for r in range(reps):
            flush.fill_(r)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            h.decode(0, q, k, v, out=out, with_lse=False)
            e1.record()
            ts.append((e0, e1))
        torch.cuda.synchronize()
        # the mean of the calls: single event intervals come in steps of ~2 us
        # on this part, which a median of a few calls would keep
        us = statistics.fmean(a.elapsed_time(b) for a, b in ts) * 1e3
        byts = 2 * wl.Hkv * N * wl.d * 2 + (2 * n * wl.Hq + 2 * n * wl.Hkv) * wl.d * 2
        flops = 4 * wl.Hq * wl.d * (n * N + n * (n + 1) // 2)
        gbs = byts / us / 1e3
        tflops = flops / us / 1e6
        t_hbm = byts / (peaks["hbm_gbs"] * 1e3)       # us at the HBM peak
        t_tc = flops / (peaks["bf16_tflops"] * 1e6)   # us at the bf16 tensor peak
        res["per_n_text"][n] = {"us": round(us, 2), "bytes": byts, "gbs": round(gbs, 1),
                                "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                "flops": flops, "tflops": round(tflops, 1),
                                "frac_of_tensor": round(tflops / peaks["bf16_tflops"], 4),
                                "bound": "hbm" if t_hbm >= t_tc else "tensor",
                                "frac": round(max(t_hbm, t_tc) / us, 4)}
    res["peak_gbs"] = peaks["hbm_gbs"]
    res["peak_tflops"] = peaks["bf16_tflops"]
    res["peak_source"] = f"{src} (copy; bf16 burst)"
    return res


def run_flatness(args):
    """8B-class layer over all 512 frames: per-frame latency vs frame index."""
    from kv_cache_selection_b200 import statekv as SKV
    rep, dec = flatness_report(SKV, Syn.workload("8b_layer"), torch.device("cuda"))
    return dict(report="flatness", decode=dec, **rep)


def run_diagnostics(args):
    """Appendix-A diagnostics on the synthetic sink recipe (1B-class layer
    shape): concentration, candidate-pool recall and retention from a
    no-eviction handle, and the historical mass that the score-based C and the
    recency C capture at the same budget.  Timing-free report."""
    import numpy as np
    from kv_cache_selection_b200 import diagnostics as Dg
    from kv_cache_selection_b200 import statekv as SKV
    wl = Syn.workload("1b_layer", frames=args.diag_frames)
    dev = torch.device("cuda")
    n_tok = wl.frames * wl.T
    full = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, n_tok, max_frames=wl.frames, dtype=wl.dtype)
    B = args.diag_b
    sel = {name: SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, B, max_frames=wl.frames, dtype=wl.dtype, select=mode)
           for name, mode in (("statekv", "global"), ("recency", "recency"))}
    steps, kept = [], {name: [] for name in sel}
    for n in range(wl.frames):
        q, k, v, pos = (t.to(dev) for t in Syn.gen_frame(wl, n))
        C = full.get_compressed(0) if n > 0 else None
        hist_pos = C["pos"][0, 0, :C["len"]].cpu().numpy() if C is not None else np.zeros(0, np.int32)
        for name, h in sel.items():
            Cs = h.get_compressed(0) if n > 0 else None
            kept[name].append(Cs["pos"][0, 0, :Cs["len"]].cpu().numpy().copy() if Cs is not None else None)
            h.prefill_frame(0, q, k, v, pos)
        full.prefill_frame(0, q, k, v, pos)
        torch.cuda.synchronize()
        stats = full.step_stats()
        L = stats["pool_len"]
        steps.append(dict(pos=np.concatenate([hist_pos, pos.cpu().numpy()]).astype(np.int64),
                          mass=stats["pool_score"][0, 0, :L].double().cpu().numpy(),
                          frame_pos=pos.cpu().numpy().astype(np.int64)))
    rep = Dg.stream_report(steps, budgets=args.diag_budgets, retained=kept)
    out = {"report": "diagnostics", "workload": f"1b_layer shape, {wl.frames} frames, sinks recipe",
           "budget_of_retained_sets": B,
           "concentration": rep["concentration"], "weighted_pool_recall": rep["weighted_recall"],
           "pool_recall": rep["recall"], "retention": rep["retention"],
           "captured_historical_mass": rep["captured"]}
    for h in list(sel.values()) + [full]:
        h.close()
    return out


def run_stack(args):
    """28 independent 8B-class layers over 128 frames.  In-order schedule:
    every frame runs its layers in order on one stream (per-frame latency vs
    frame index).  Pipelined schedule: frames alternate over `--stack-pipeline`
    streams and layer l of frame n+1 waits only for layer l of frame n (an
    event per layer), so frame n+1's early layers overlap frame n's later
    ones; reported as frames/s per layer over the same frames."""
    from kv_cache_selection_b200 import statekv as SKV
    wl = Syn.workload("8b_stack")
    dev = torch.device("cuda")
    n_frames = args.stack_frames or wl.frames
    layers = [Syn.gen_frames_device(wl, n_frames, layer=l, device=dev) for l in range(wl.layers)]
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    fill = math.ceil(wl.B / wl.T)
    d_bytes = wl.layers * n_frames * wl.T * wl.Hkv * wl.d * 2 * 2

    # in order, one stream, per-frame events
    h = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=n_frames, dtype=wl.dtype)
    h.reserve_layers(wl.layers)
    out = torch.empty_like(layers[0][0][0])

    def frame(n):
        for l, (q, k, v, pos) in enumerate(layers):
            h.prefill_frame(l, q[n], k[n], v[n], pos[n], out)

    us = _per_frame_times(frame, n_frames, flush, dev)
    h.close()
    flat = _flatness(us, fill)
    rep = {"report": "stack", "workload": f"8b_stack: {wl.layers} layers x {n_frames} frames, B={wl.B}",
           "in_order": {"per_frame_us_all_layers": flat,
                        "per_frame_layer_us": round(flat["p50_us"] / wl.layers, 2),
                        "frames_per_s_per_layer": round(1e6 / (flat["p50_us"] / wl.layers), 1),
                        "per_frame_us_every_8": [round(x, 1) for x in us[::8]]},
           "detailed_state_bytes_K_plus_V": d_bytes}

    # whole-run throughput of the steady-state frames, L2 not flushed (frames
    # overlap in the pipelined schedule): one stream (in order) against P
    # streams (pipelined)
    main = torch.cuda.current_stream()

    def whole_run(P):
        h = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=n_frames, dtype=wl.dtype)
        h.reserve_layers(wl.layers)
        streams = [torch.cuda.Stream(device=dev) for _ in range(P)]
        outs = [torch.empty_like(out) for _ in range(P)]
        layer_done = [torch.cuda.Event() for _ in range(wl.layers)]

        def run_frames(n0, n1):
            for n in range(n0, n1):
                st = streams[n % P]
                for l, (q, k, v, pos) in enumerate(layers):
                    st.wait_event(layer_done[l])          # frame n-1 of layer l is done
                    h.prefill_frame(l, q[n], k[n], v[n], pos[n], outs[n % P], stream=st)
                    layer_done[l].record(st)

        for st in streams:
            st.wait_stream(main)
        run_frames(0, fill)                               # fill C (not timed)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for st in streams:
            st.wait_stream(main)
        run_frames(fill, n_frames)
        for st in streams:
            main.wait_stream(st)
        e1.record(main)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        h.close()
        steady = n_frames - fill
        return {"streams": P, "frames_timed": steady, "per_frame_us_all_layers": round(ms * 1e3 / steady, 1),
                "per_frame_layer_us": round(ms * 1e3 / steady / wl.layers, 2),
                "frames_per_s_per_layer": round(steady * wl.layers / (ms / 1e3), 1)}

    rep["whole_run_unflushed"] = {"in_order": whole_run(1), "pipelined": whole_run(max(2, args.stack_pipeline))}
    return rep


def sweep_report(frames_list, b_list, dev):
    """8B layer shape, 4 streams per launch: cumulative StateKV prefill device
    time over the first N frames against full_causal_prefill over the same
    N*256 tokens (one batched call, 4 sequences), and the first N on the grid
    where StateKV is cheaper (the compute crossover)."""
    from kv_cache_selection_b200 import statekv as SKV
    wl = Syn.workload("8b_sweep")
    S = wl.streams
    n_max = max(frames_list)
    per = [Syn.gen_frames_device(wl, n_max, stream=s, device=dev) for s in range(S)]
    # [S][n][T][H][d] so that the first N frames of a stream are one sequence
    Q = torch.stack([p[0] for p in per])
    Kt = torch.stack([p[1] for p in per])
    V = torch.stack([p[2] for p in per])
    P = torch.stack([p[3] for p in per])
    del per
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    res = {"workload": f"8b layer shape, {S} streams per launch, frames {list(frames_list)}",
           "statekv": {}, "full_causal_us": {}, "crossover_frames": {}, "analytic_crossover_frames_3_passes": {}}
    fc = {}
    for N in frames_list:
        ntok = N * wl.T
        q = Q[:, :N].reshape(S, ntok, wl.Hq, wl.d).contiguous()
        kk = Kt[:, :N].reshape(S, ntok, wl.Hkv, wl.d).contiguous()
        vv = V[:, :N].reshape(S, ntok, wl.Hkv, wl.d).contiguous()
        out = torch.empty_like(q)
        SKV.full_causal_prefill(q, kk, vv, out=out, with_lse=False)  # warm-up
        torch.cuda.synchronize()
        _flush_l2(flush, N)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        SKV.full_causal_prefill(q, kk, vv, out=out, with_lse=False)
        e1.record()
        torch.cuda.synchronize()
        fc[N] = e0.elapsed_time(e1) * 1e3
        res["full_causal_us"][N] = round(fc[N], 1)
        del out, q, kk, vv
    for B in b_list:
        h = SKV.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, B, max_frames=n_max, dtype=wl.dtype, n_streams=S)
        h.reserve_layers(1)
        qs = torch.empty((S, wl.T, wl.Hq, wl.d), dtype=wl.torch_dtype, device=dev)
        ks = torch.empty((S, wl.T, wl.Hkv, wl.d), dtype=wl.torch_dtype, device=dev)
        vs = torch.empty_like(ks)
        ps = torch.empty((S, wl.T), dtype=torch.int32, device=dev)
        out = torch.empty_like(qs)
        times = []
        for n in range(n_max):
            qs.copy_(Q[:, n]); ks.copy_(Kt[:, n]); vs.copy_(V[:, n]); ps.copy_(P[:, n])
            _flush_l2(flush, n)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            h.prefill_frame(0, qs, ks, vs, ps, out)
            e1.record()
            times.append((e0, e1))
        torch.cuda.synchronize()
        us = [a.elapsed_time(b) * 1e3 for a, b in times]
        cum, acc = {}, 0.0
        for n, t in enumerate(us):
            acc += t
            if n + 1 in frames_list:
                cum[n + 1] = round(acc, 1)
        fill = math.ceil(B / wl.T)
        res["statekv"][B] = {"cumulative_us": cum, "steady_step_us_4_streams": _flatness(us, fill)["p50_us"]}
        cross = None
        for N in sorted(frames_list):
            if cum[N] <= fc[N]:
                cross = N
                break
        res["crossover_frames"][B] = cross
        res["analytic_crossover_frames_3_passes"][B] = round(3 * (B + wl.T / 2) / wl.T, 1)
        h.close()
    del Q, Kt, V, P
    return res


def run_sweep(args):
    return dict(report="sweep", **sweep_report(args.sweep_frames, args.sweep_b, torch.device("cuda")))


# ------------------------------------------------------------ reference arm --
def run_reference(args, wl):
    rank, _, world = rank_info()
    if rank != 0:
        return
    from threadpoolctl import threadpool_info
    from oracle import statekv_oracle as O

    K, W = args.steps, args.warmup
    G = wl.Hq // wl.Hkv
    # steady state needs a full C: build it from the oracle's own fill frames on
    # one KV head group (this prologue is not timed)
    kvh = 1
    fill = math.ceil(wl.B / wl.T)
    n_distinct = min(args.distinct_frames, fill + W + K, 32)
    frames = Syn.gen_frames(wl, n_distinct)
    st = O.LayerState.empty(kvh, wl.d)
    for n in range(fill):
        q, k, v, _ = frames[n % n_distinct]
        pos = torch.arange(n * wl.T, (n + 1) * wl.T).numpy()
        st, _ = O.statekv_step(st, q[:, :kvh * G], k[:, :kvh], v[:, :kvh], pos, wl.B)
    t_steps = []
    n = fill
    for j in range(W + K):
        q, k, v, _ = frames[n % n_distinct]
        pos = torch.arange(n * wl.T, (n + 1) * wl.T).numpy()
        t0 = time.perf_counter()
        st, _ = O.statekv_step(st, q[:, :kvh * G], k[:, :kvh], v[:, :kvh], pos, wl.B)
        dt = time.perf_counter() - t0
        if j >= W:
            t_steps.append(dt)
        n += 1
    frac = kvh / wl.Hkv
    total = sum(t_steps) / frac        # scaled to all KV heads
    value = K / total
    threads = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
    cores = int(max(threads) if threads else 1)
    sample = (f"each step: one float64 oracle step of {wl.name} in steady state on {kvh} of {wl.Hkv} "
              f"KV heads ({kvh * G} query heads), time scaled by {wl.Hkv}/{kvh}")
    line = {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(total / K * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{wl.name}: Hq={wl.Hq} Hkv={wl.Hkv} d={wl.d} T={wl.T} B={wl.B}, "
                                   f"steady state (C full), frame-causal, global select",
                       "global_batch": 1, "seq_len": wl.T, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "host_cpus": os.cpu_count(), "sample": sample},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="8b_layer", choices=sorted(Syn.WORKLOADS))
    ap.add_argument("--l2", choices=["flush", "resident"], default="flush")
    ap.add_argument("--distinct-frames", type=int, default=96,
                    help="distinct synthetic frames kept on the device (cycled)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flatness", action="store_true", help="skip the 512-frame flatness pass")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle time")
    ap.add_argument("--mode", choices=["headline", "flatness", "stack", "sweep", "diagnostics"], default="headline",
                    help="headline: the contract's JSON line; others: report lines")
    ap.add_argument("--stack-frames", type=int, default=0)
    ap.add_argument("--stack-pipeline", type=int, default=4, help="streams of the pipelined stack schedule")
    ap.add_argument("--diag-frames", type=int, default=64)
    ap.add_argument("--diag-b", type=int, default=1024, help="budget of the retained sets compared")
    ap.add_argument("--diag-budgets", type=int, nargs="+", default=[1, 16, 256, 1024, 4096])
    ap.add_argument("--sweep-frames", type=int, nargs="+", default=[32, 64, 128, 256, 512, 1024])
    ap.add_argument("--sweep-b", type=int, nargs="+", default=[1024, 2048, 4096])
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = Syn.workload(args.workload)
    if args.mode != "headline":
        clocks = ClockSampler(0)
        clocks.start()
        rep = {"flatness": run_flatness, "stack": run_stack, "sweep": run_sweep,
               "diagnostics": run_diagnostics}[args.mode](args)
        rep["clocks"] = clocks.stop()
        print(json.dumps(rep), flush=True)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
