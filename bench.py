"""Benchmark of the sparse absorbed MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
                    [--no-extras] [--sets S]

One step = one call of the whole decode path (absorb, sparse attend, combine +
value-up) over one batch of B rows.  The default workload is the B=64,
32K-context, top-2048 configuration.  Inputs are synthetic (seeded), generated
on the host in bf16 and kept resident in HBM; independent input sets
(queries, index sets, end positions and a separate copy of wkv_b each, and the
caches too when they are small) rotate between steps, enough of them that one
rotation moves more than twice the L2 size, so a step never finds the
previous step's bytes in L2.

The timed region is a window of exactly K steps, bracketed by a barrier and a
synchronize; windows are repeated until they span at least 0.5 s and the
median window gives the step time (with NVML clock samples from all of them).
The same line carries per-kernel cold timings, every other configuration of
the pages (``per_config``), the output projection, the sparse prefill and the
end-to-end figure through the host-buffer entry point.

Prints one JSON line (rank 0).  Under torchrun every rank runs its own batch
(weak scaling, no collective on the path); the step time is the maximum over
ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
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
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_latent_attention_absorb_b200 import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "b64_ctx1k-32k_top2048"
NSETS = 4
METRIC = "sparse MLA decode queries/s"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def algorithmic(B, K, sum_k):
    """Bytes and FLOPs the method must move / compute for one call (no dense
    mask, no split partials): wkv_b once, the queries, the gathered latent +
    rotary rows of every selected position, the indices, end_pos and out."""
    bytes_ = (128 * 256 * 512 * 2 + B * 128 * (128 + 64) * 2 + 1152 * sum_k + 4 * B * K + 4 * B + B * 128 * 128 * 2)
    flops = 2 * 128 * 128 * 512 * 2 * B + 2 * 128 * (576 + 512) * sum_k
    return bytes_, flops


def attend_bytes(B, K, sum_k):
    """Algorithmic bytes of the sparse-attend kernel alone: the gathered rows
    (1152 B per selected position), the indices and end_pos."""
    return 1152 * sum_k + 4 * B * K + 4 * B


def source_hash():
    h = hashlib.sha256()
    for f in ("kernels.cuh", "ptx.cuh", "mla_sparse_decode.cu"):
        with open(os.path.join(ROOT, "sparse_latent_attention_absorb_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds, all of them get the maximum (a no-op with one rank).  Every
    rank must call it at the same point (it is a collective)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(rows_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Queries per second of the whole job: every rank decodes its own batch
    of rows_per_rank rows per step (weak scaling, replicas), timed by the
    slowest rank."""
    return rows_per_rank * world * steps / (ms / 1e3)


def ncu_traffic(workload):
    """DRAM bytes per launch of the sparse-attend kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("source_hash") == source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML by a background
    thread as fast as NVML answers, kept only between mark_start() and
    mark_end() (the host brackets the timed region with them: it enqueues the
    steps and then blocks until they finish).  Falls back to nvidia-smi at
    100 ms if NVML is unavailable."""

    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"))

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []  # (host time, sm MHz, set of reasons)
        self.t0 = self.t1 = None
        self.max_mhz = None
        self._stop = False

    def _nvml_handle(self, nvml):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return nvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _run(self):
        nvml = self.nvml
        bits = [(name, getattr(nvml, "nvmlClocksEventReason" + suffix, 0)) for name, suffix in self.REASONS]
        get_reasons = getattr(nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop and len(self.samples) < 200000:
            try:
                mhz = nvml.nvmlDeviceGetClockInfo(self.h, nvml.NVML_CLOCK_SM)
                mask = get_reasons(self.h)
            except Exception:
                break
            self.samples.append((time.perf_counter(), float(mhz), {n for n, b in bits if mask & b}))

    def __enter__(self):
        import threading
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = self._nvml_handle(pynvml)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:
            self.nvml = None
            self._smi_start()
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self._stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)
        else:
            self._smi_stop()
        return False

    # nvidia-smi fallback (100 ms period)
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def _smi_start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def _smi_stop(self):
        if getattr(self, "proc", None) is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        now = time.perf_counter()
        for ln in out.splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                mhz, self.max_mhz = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            reasons = {n for (n, _), v in zip(self.REASONS, parts[2:6]) if v.lower() == "active"}
            self.samples.append((now, mhz, reasons))  # times unknown: kept as one window

    def summary(self):
        if self.thread is not None and self.t0 is not None and self.t1 is not None:
            inside = [s for s in self.samples if self.t0 <= s[0] <= self.t1]
        else:
            inside = list(self.samples)
        mhz = [s[1] for s in inside]
        reasons = set().union(*[s[2] for s in inside]) if inside else set()
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz),
                "source": "nvml, inside the timed region" if self.thread is not None else "nvidia-smi"}


# ----------------------------------------------------------------------------- GPU arm

L2_BYTES = 126 * 2 ** 20  # B200 L2 (the footprint rule below keeps a rotation at > 2x this)


def n_rotating_sets(w, floor=NSETS):
    """Input sets to rotate so that one rotation touches more than twice the
    L2 size: each set holds its own wkv_b copy, queries, indices and, when the
    workload's caches are small enough to stay in L2, its own caches."""
    per_set = 128 * 256 * 512 * 2 + w.B * 128 * 192 * 2 + 4 * w.B * w.K
    if own_caches(w):
        per_set += w.B * w.S_max * 1152
    return max(floor, math.ceil(2 * L2_BYTES / per_set))


def own_caches(w):
    """Caches smaller than twice L2 are drawn per input set (else the gathered
    rows of one step would still be in L2 at the next)."""
    return w.B * w.S_max * 1152 < 2 * L2_BYTES


def make_sets(w, device, n_sets):
    """n_sets input sets on the device.  Large caches are shared (model
    state); queries, indices, end positions and a wkv_b copy are drawn per
    set, and small caches too."""
    base = wl.generate(w)
    shared = None if own_caches(w) else {k: base[k].to(device) for k in ("kv_cache", "pe_cache")}
    sets = []
    for i in range(n_sets):
        d = base if i == 0 else wl.generate(w, seed_offset=i, caches=shared is None)
        keys = ("q_nope", "q_pe", "end_pos", "topk_idx", "wkv_b") + (("kv_cache", "pe_cache") if shared is None else ())
        s = {k: d[k].to(device) for k in keys}
        if shared is not None:
            s.update(shared)
        s["scale"] = d["scale"]
        s["sum_k"] = wl.selected_count(d["end_pos"], d["topk_idx"])
        s["host"] = d
        sets.append(s)
    return sets, base


def call_roofline(B, K, sum_k, ms_per_call):
    hbm, tf, _, kind = peaks()
    call_bytes, call_flops = algorithmic(B, K, sum_k)
    t_hbm = call_bytes / (hbm * 1e9)
    t_tc = call_flops / (tf * 1e12)
    roof_ms = max(t_hbm, t_tc) * 1e3
    return {"alg_bytes": call_bytes, "alg_flops": call_flops, "t_hbm_ms": t_hbm * 1e3, "t_tensor_ms": t_tc * 1e3,
            "roofline_ms": roof_ms, "frac": roof_ms / ms_per_call, "bound": "hbm" if t_hbm >= t_tc else "tensor",
            "peaks": {"hbm_gbs": hbm, "bf16_tflops": tf, "source": kind}}


class Decoder:
    """One graph-captured decode call per input set, and one graph of all the
    sets' calls back to back (a replay = len(sets) steps)."""

    def __init__(self, lib, w, sets, device, stream):
        import ctypes
        self.lib, self.w, self.sets, self.stream = lib, w, sets, stream
        self.ws = torch.empty(lib.mla_sparse_decode_workspace_size(w.B, w.K, w.S_max), dtype=torch.uint8,
                              device=device)
        self.outs = [torch.empty((w.B, 128, 128), dtype=torch.bfloat16, device=device) for _ in sets]
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

        def call(i, st):
            s = sets[i]
            rc = lib.mla_sparse_decode(P(s["q_nope"]), P(s["q_pe"]), P(s["kv_cache"]), P(s["pe_cache"]),
                                       P(s["end_pos"]), P(s["topk_idx"]), P(s["wkv_b"]), ctypes.c_float(s["scale"]),
                                       P(self.outs[i]), w.B, w.K, w.S_max, P(self.ws), self.ws.numel(), None, None,
                                       ctypes.c_void_p(st.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"mla_sparse_decode: status {rc}")

        with torch.cuda.stream(stream):
            for i in range(len(sets)):
                call(i, stream)
        stream.synchronize()
        self.graphs = []
        for i in range(len(sets)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                call(i, torch.cuda.current_stream())
            self.graphs.append(g)
        self.chain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.chain, stream=stream):
            for i in range(len(sets)):
                call(i, torch.cuda.current_stream())
        torch.cuda.synchronize()

    def run(self, n):
        """n decode steps, input sets in rotation."""
        n_sets = len(self.sets)
        with torch.cuda.stream(self.stream):
            for _ in range(n // n_sets):
                self.chain.replay()
            for i in range(n % n_sets):
                self.graphs[i].replay()

    def time_ms(self, n):
        """Device time of n steps (CUDA events on the launching stream)."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        self.run(n)
        e1.record(self.stream)
        self.stream.synchronize()
        return e0.elapsed_time(e1)

    def release(self):
        self.graphs.clear()
        self.chain = None


def per_config(lib, device, stream, min_s=0.1):
    """Every workload of the pages' configurations (the dense pass included),
    each timed from graphs of back-to-back decode calls with its own rotating
    input sets, with its whole-call roofline."""
    out = {}
    for name, w in wl.WORKLOADS.items():
        sets, _ = make_sets(w, device, n_rotating_sets(w))
        dec = Decoder(lib, w, sets, device, stream)
        dec.run(2 * len(sets))
        n = len(sets)
        t = dec.time_ms(n)
        reps = max(1, math.ceil(min_s * 1e3 / max(t, 1e-3)))
        ms = dec.time_ms(n * reps) / (n * reps)
        sum_k = statistics.mean(s["sum_k"] for s in sets)
        out[name] = {"B": w.B, "K": w.K, "S_max": w.S_max, "sum_k_mean": sum_k, "splits": lib.mla_num_splits(w.B, w.K),
                     "ms_per_call": ms, "queries_per_s": w.B / (ms * 1e-3), "calls_timed": n * reps,
                     "rotating_sets": n, "own_caches_per_set": own_caches(w),
                     "call_roofline": call_roofline(w.B, w.K, sum_k, ms)}
        dec.release()
        del dec, sets
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def gpu_arm(args, rank, world, device):
    import ctypes

    import sparse_latent_attention_absorb_b200 as pkg
    from sparse_latent_attention_absorb_b200 import binding

    lib = pkg.load_library()
    w = wl.ALL_WORKLOADS[args.workload]
    sets, base = make_sets(w, device, args.sets or n_rotating_sets(w))
    B, K, S_max = w.B, w.K, w.S_max
    n_split = pkg.num_splits(B, K)
    stream = torch.cuda.Stream(device=device)
    dec = Decoder(lib, w, sets, device, stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- timed region: windows of exactly K decode steps, each bracketed by
    # a barrier and a synchronize, repeated until the windows span >= 0.5 s;
    # the median window (max over ranks) gives the step time
    dec.run(args.warmup)
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    probe = max_over_ranks(dec.time_ms(args.steps), world, device)
    repeats = max(1, min(100000, math.ceil(500.0 / max(probe, 1e-3))))
    windows = []
    with ClockSampler(torch.cuda.current_device() if device.index is None else device.index) as clocks:
        clocks.mark_start()
        for _ in range(repeats):
            barrier()
            torch.cuda.synchronize()
            windows.append(max_over_ranks(dec.time_ms(args.steps), world, device))
        clocks.mark_end()
    barrier()
    torch.cuda.synchronize()
    window_ms = statistics.median(windows)
    ms_per_step = window_ms / args.steps
    value = whole_job_rate(B, world, args.steps, window_ms)
    launches = 3 * args.steps

    # ---- per-kernel live timing, cold: graphs of back-to-back launches of one
    # kernel on the same stream, input sets rotating, and for the two kernels
    # that read only half of wkv_b each, enough wkv_b copies that a rotation of
    # the halves they read exceeds L2
    q_lat = [torch.empty((B, 128, 512), dtype=torch.bfloat16, device=device) for _ in sets]
    # the attention kernel's per-split output (bf16; the mixed latent itself
    # when each row is a single split)
    o_part = torch.empty((B, n_split, 128, 512), dtype=torch.bfloat16, device=device)
    lse_part = torch.empty((B, n_split, 128), dtype=torch.float32, device=device)
    n_w = max(len(sets), math.ceil(2 * L2_BYTES / (128 * 128 * 512 * 2)))
    w_copies = [sets[i]["wkv_b"] if i < len(sets) else torch.empty_like(sets[0]["wkv_b"]).copy_(sets[i % len(sets)]["wkv_b"])
                for i in range(n_w)]
    sv = ctypes.c_void_p(stream.cuda_stream)
    ns = len(sets)

    def k_absorb(r):
        return lib.mla_absorb_q(P(sets[r % ns]["q_nope"]), P(w_copies[r % n_w]), P(q_lat[r % ns]), B, sv)

    def k_attend(r):
        s = sets[r % ns]
        return lib.mla_sparse_attend(P(q_lat[r % ns]), P(s["q_pe"]), P(s["kv_cache"]), P(s["pe_cache"]),
                                     P(s["end_pos"]), P(s["topk_idx"]), ctypes.c_float(s["scale"]), P(o_part),
                                     P(lse_part), B, K, S_max, n_split, None, sv)

    def k_combine(r):
        return lib.mla_combine_value_up(P(o_part), P(lse_part), P(w_copies[r % n_w]), P(dec.outs[r % ns]), None, B,
                                        n_split, sv)

    def time_kernel(fn, reps):
        """Device time of one launch: `reps` back-to-back launches captured in
        a CUDA graph (host launch cost excluded), the second replay timed."""
        with torch.cuda.stream(stream):
            for r in range(4):
                assert fn(r) == 0
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                fn(r)
        with torch.cuda.stream(stream):
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return e0.elapsed_time(e1) / reps

    with torch.cuda.stream(stream):
        for i in range(ns):
            k_absorb(i)
    stream.synchronize()
    reps = 4 * max(ns, n_w) * 4
    t_absorb = time_kernel(k_absorb, reps)
    t_attend = time_kernel(k_attend, reps)
    t_combine = time_kernel(k_combine, reps)
    del w_copies

    extras = {}
    if not args.no_extras:
        extras = extra_measurements(args, lib, dec, sets, w, device, stream, rank, world)

    # ---- roofline of the dominant kernel and of the whole call
    hbm, tf, tf_sus, kind = peaks()
    sum_k = statistics.mean(s["sum_k"] for s in sets)
    a_bytes = attend_bytes(B, K, sum_k)
    achieved = a_bytes / (t_attend * 1e-3) / 1e9
    traffic = ncu_traffic(args.workload)
    cr = call_roofline(B, K, sum_k, ms_per_step)

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "heads": 128, "S_max": S_max, "K": K,
                   "end_pos": list(w.end_pos), "index": w.index, "sum_k_mean": sum_k, "splits": n_split,
                   "parallelism": f"replicas x{world} (batch rows)",
                   "l2": f"{ns} rotating input sets (queries, indices, wkv_b copy each"
                         f"{', caches' if own_caches(w) else ''}); a rotation moves {ns * cr['alg_bytes'] / 1e6:.0f} MB "
                         f"> 2 x 126 MB L2",
                   "timing": (f"{repeats} windows of exactly {args.steps} steps, each bracketed by a barrier and a "
                              f"synchronize; median window ({statistics.median(windows):.3f} ms, min "
                              f"{min(windows):.3f}, max {max(windows):.3f}); windows span "
                              f"{sum(windows) / 1e3:.2f} s; CUDA graphs of consecutive steps, CUDA events on the "
                              f"launching stream"),
                   "windows": repeats},
        "roofline": {"bound": "hbm", "kernel": "sparse_attend_kernel", "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                     "peak_source": f"{kind} hbm_gbs (burst copy)", "alg_bytes_per_launch": a_bytes,
                     "ms_per_launch": t_attend},
        "call_roofline": cr,
        "kernels_ms": {"absorb": t_absorb, "sparse_attend": t_attend, "combine_value_up": t_combine,
                       "how": f"cold: graphs of {reps} back-to-back launches of one kernel, input sets rotating, "
                              f"{n_w} wkv_b copies rotating for absorb and value-up"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    res.update(extras)
    dec.release()
    return res, base


def extra_measurements(args, lib, dec, sets, w, device, stream, rank, world):
    """The other configurations, the rows after the path (output projection,
    sparse prefill) and the end-to-end figure through the host-buffer API."""
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    sv = ctypes.c_void_p(stream.cuda_stream)
    hbm = peaks()[0]
    B, K, S_max = w.B, w.K, w.S_max

    def time_graph(fn, reps):
        with torch.cuda.stream(stream):
            for r in range(2):
                assert fn(r) == 0
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                fn(r)
        with torch.cuda.stream(stream):
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return e0.elapsed_time(e1) / reps

    # ---- the step after the path: the output projection of the decode
    # outputs (page "Attention update"), wo [7168, 16384] bf16 = 235 MB, more
    # than L2, so every call streams it from HBM
    p_dim = wl.D_MODEL
    p_wo = wl.generate_projection(1, p_dim, seed=5001)["wo"].to(device)
    p_delta = torch.empty((B, p_dim), dtype=torch.bfloat16, device=device)
    p_ws = torch.empty(lib.mla_output_projection_workspace_size(B, p_dim), dtype=torch.uint8, device=device)

    def k_project(r):
        return lib.mla_output_projection(P(dec.outs[r % len(sets)]), P(p_wo), P(p_delta), B, p_dim, P(p_ws),
                                         p_ws.numel(), None, sv)

    # the same projection from the prepared copy of wo (built once per weight,
    # outside the timed region): each work unit's weights are one contiguous
    # 64 KB read
    p_prep = torch.empty(p_dim * 16384, dtype=torch.bfloat16, device=device)
    assert lib.mla_prepare_wo(P(p_wo), 16384, p_dim, 16384, P(p_prep), sv) == 0

    def k_project_prepared(r):
        return lib.mla_output_projection_prepared(P(dec.outs[r % len(sets)]), P(p_prep), P(p_delta), B, p_dim,
                                                  16384, P(p_ws), p_ws.numel(), None, sv)

    t_project_in_place = time_graph(k_project, 50)
    t_project = time_graph(k_project_prepared, 50)
    p_bytes = p_dim * 16384 * 2 + B * 16384 * 2 + B * p_dim * 2
    del p_wo, p_prep

    # ---- the sparse prefill (page "Queries", prefill mode): one sequence of
    # 4096 positions, top-2048, one row per query position reading the
    # chunk's own latents (4.7 MB: they stay in L2)
    pf = wl.generate_prefill(1, 4096, 2048, seed=5101)
    pf_sel = int(((pf["topk_idx"] >= 0) & (pf["topk_idx"] < pf["end_pos"].unsqueeze(1))).sum())
    pfd = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in pf.items()}
    R_pf, K_pf, S_pf = pf["q_nope"].shape[0], pf["topk_idx"].shape[1], pf["kv_cache"].shape[1]
    pf_out = torch.empty((R_pf, 128, 128), dtype=torch.bfloat16, device=device)
    pf_ws = torch.empty(lib.mla_sparse_decode_workspace_size(R_pf, K_pf, S_pf), dtype=torch.uint8, device=device)

    def k_prefill(r):
        return lib.mla_sparse_prefill(P(pfd["q_nope"]), P(pfd["q_pe"]), P(pfd["kv_cache"]), P(pfd["pe_cache"]),
                                      P(pfd["cache_slot"]), P(pfd["end_pos"]), P(pfd["topk_idx"]), P(pfd["wkv_b"]),
                                      ctypes.c_float(pfd["scale"]), P(pf_out), R_pf, K_pf, S_pf, 1, P(pf_ws),
                                      pf_ws.numel(), None, None, sv)

    t_prefill = time_graph(k_prefill, 5)
    del pfd, pf_out, pf_ws

    extras = {
        "projection": {"what": "output projection delta = x . wo^T of the decode outputs, wo bf16 [7168, 16384], "
                               "from the prepared wo (mla_output_projection_prepared)",
                       "ms_per_call": t_project, "launches_per_call": 1 if p_ws.numel() <= 256 else 2,
                       "ms_per_call_in_place": t_project_in_place,
                       "roofline": {"bound": "hbm", "achieved": p_bytes / (t_project * 1e-3) / 1e9, "peak": hbm,
                                    "unit": "GB/s", "frac": p_bytes / (t_project * 1e-3) / 1e9 / hbm,
                                    "alg_bytes_per_call": p_bytes, "peak_source": "measured hbm_gbs"}},
        "prefill": {"what": "sparse prefill of one 4096-position sequence, top-2048, causal: one row per query "
                            "position (mla_sparse_prefill)", "ms_per_call": t_prefill,
                    "tokens_per_s": R_pf / (t_prefill * 1e-3), "selected_positions": pf_sel,
                    "gathered_GBps": pf_sel * 1152 / (t_prefill * 1e-3) / 1e9},
    }

    # ---- end to end through the public API with host buffers
    extras["e2e"] = e2e_measurement(args, dec, sets, w, device, stream, world)

    # ---- every configuration of the pages, each with its own roofline
    extras["per_config"] = per_config(lib, device, stream)
    return extras


def e2e_measurement(args, dec, sets, w, device, stream, world, n_streams=3):
    """Per step one call of the C ABI's host-buffer entry point (through the
    Python binding): the step's queries, end positions and indices are
    uploaded from pinned host memory, the decode runs and the result is read
    back to pinned host memory, all on the call's stream.  Steps rotate over
    n_streams streams, each with its own workspace and output buffer, so the
    uploads and read-backs of neighbouring steps overlap this step's kernels."""
    import sparse_latent_attention_absorb_b200 as api
    B, K, S_max = w.B, w.K, w.S_max
    from sparse_latent_attention_absorb_b200 import binding
    names = ("q_nope", "q_pe", "end_pos", "topk_idx")
    # each set's inputs in one pinned buffer laid out like the staging area:
    # the entry point uploads them in one copy
    hins, hbufs = [], []
    for s_ in sets:
        hbuf, views = binding.host_input_buffer(B, K, S_max)
        for k in names:
            views[k].copy_(s_["host"][k])
        hins.append(views)
        hbufs.append(hbuf)
    houts = [torch.empty((B, 128, 128), dtype=torch.bfloat16).pin_memory() for _ in range(n_streams)]
    hws = [torch.empty(api.host_workspace_size(B, K, S_max), dtype=torch.uint8, device=device)
           for _ in range(n_streams)]
    streams = [stream] + [torch.cuda.Stream(device=device) for _ in range(n_streams - 1)]
    h2d = sum(hins[0][k].numel() * hins[0][k].element_size() for k in names)
    d2h = houts[0].numel() * houts[0].element_size()

    def step(i):
        k, si = i % n_streams, i % len(sets)
        h = hins[si]
        api.mla_sparse_decode_host(h["q_nope"], h["q_pe"], h["end_pos"], h["topk_idx"], sets[si]["kv_cache"],
                                   sets[si]["pe_cache"], sets[si]["wkv_b"], sets[si]["scale"], houts[k], hws[k],
                                   stream=streams[k])

    def window(n):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(streams[0])
        for s_ in streams[1:]:
            s_.wait_event(f0)
        for it in range(n):
            step(it)
        for s_ in streams[1:]:
            done = torch.cuda.Event()
            done.record(s_)
            streams[0].wait_event(done)
        f1.record(streams[0])
        torch.cuda.synchronize()
        return f0.elapsed_time(f1)

    for it in range(max(50, args.warmup)):  # host-side paths warm as well
        step(it)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    probe = max_over_ranks(window(args.steps), world, device)
    repeats = max(1, min(10000, math.ceil(500.0 / max(probe, 1e-3))))
    wins = [max_over_ranks(window(args.steps), world, device) for _ in range(repeats)]
    e_ms = statistics.median(wins)
    ceiling = copy_ceiling(args, hbufs, houts, streams, world, device)
    ceiling["frac"] = whole_job_rate(B, world, args.steps, e_ms) / ceiling["value"]
    return {"value": whole_job_rate(B, world, args.steps, e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "windows": repeats, "copy_bound": ceiling,
            "how": f"per step one mla_sparse_decode_host call (the step's inputs uploaded from one pinned host "
                   f"buffer in one copy, decode, result read back to pinned memory, all on the call's stream); "
                   f"steps rotate over {n_streams} streams; median of {repeats} windows of {args.steps} steps"}


def copy_ceiling(args, hbufs, houts, streams, world, device):
    """What the copies allow: the step's packed input upload (pinned host ->
    device, one copy) and its output read-back (device -> pinned host), timed
    back to back with no kernels, each direction alone and both at once on two
    streams.  The upload is the larger of the two, so a step can take no less
    than the upload alone: `value` is that rate in queries/s, the ceiling of
    the end-to-end figure whatever the kernels do (frac = end to end / it)."""
    n = max(args.steps, 50)
    up_bytes, down_bytes = hbufs[0].numel(), houts[0].numel() * houts[0].element_size()
    dev_in = [torch.empty(up_bytes, dtype=torch.uint8, device=device) for _ in range(2)]
    dev_out = torch.empty(down_bytes, dtype=torch.uint8, device=device)
    outs = [o.view(torch.uint8).view(-1) for o in houts]
    s_up, s_down = streams[0], streams[1]

    def run(up: bool, down: bool) -> float:
        ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in ("u", "d")}
        start = torch.cuda.Event()
        start.record(s_up)
        s_down.wait_event(start)
        ev["u"][0].record(s_up)
        ev["d"][0].record(s_down)
        for i in range(n):
            if up:
                with torch.cuda.stream(s_up):
                    dev_in[i % 2].copy_(hbufs[i % len(hbufs)], non_blocking=True)
            if down:
                with torch.cuda.stream(s_down):
                    outs[i % len(outs)].copy_(dev_out, non_blocking=True)
        ev["u"][1].record(s_up)
        ev["d"][1].record(s_down)
        torch.cuda.synchronize()
        t = max(ev["u"][0].elapsed_time(ev["u"][1]) if up else 0.0, ev["d"][0].elapsed_time(ev["d"][1]) if down else 0.0)
        return max_over_ranks(t, world, device) / n

    for _ in range(3):
        run(True, True)
    up_ms = statistics.median(run(True, False) for _ in range(5))
    down_ms = statistics.median(run(False, True) for _ in range(5))
    both_ms = statistics.median(run(True, True) for _ in range(5))
    B = houts[0].shape[0]
    return {"value": whole_job_rate(B, world, 1, up_ms), "unit": UNIT, "upload_ms_per_step": up_ms,
            "readback_ms_per_step": down_ms, "both_ms_per_step": both_ms,
            "h2d_gbs": up_bytes / up_ms / 1e6, "d2h_gbs": down_bytes / down_ms / 1e6,
            "how": f"{n} copies back to back, no kernels: the {up_bytes}-byte packed upload alone (value), the "
                   f"{down_bytes}-byte read-back alone, and both at once on two streams (both_ms_per_step)"}


# ----------------------------------------------------------------------------- CPU oracle

def cpu_baseline(args, base, budget_s=12.0):
    """The fp64 oracle as it stands on a bounded sample of the same workload:
    whole batch rows (all 128 heads), repeated passes until about budget_s of
    CPU work."""
    import oracle
    w = wl.ALL_WORKLOADS[args.workload]
    d = base
    run = lambda rows: oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"],  # noqa: E731
                                                d["end_pos"], d["topk_idx"], d["wkv_b"], d["scale"], rows=rows)
    t0 = time.perf_counter()
    run([0])
    t1 = max(time.perf_counter() - t0, 1e-4)
    per_pass = min(w.B, max(1, int(budget_s / t1)))
    rows = list(range(per_pass))
    done, t_total, passes = 0, 0.0, 0
    while t_total < budget_s * 0.8 and passes < 1000:
        t0 = time.perf_counter()
        run(rows)
        t_total += time.perf_counter() - t0
        done += len(rows)
        passes += 1
    return {"value": done / t_total, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{passes} pass(es) over {len(rows)} of {w.B} batch rows (all 128 heads): "
                      f"{done} rows in {t_total:.1f} s"}


def reference_arm(args, rank, world, budget_s=90.0):
    """The oracle as it stands on the host cores.  A step is one batch row of
    the workload, or, when K such steps would not fit in about budget_s, a
    fixed subset of that row's heads sized so they do (the oracle is
    dimension-generic; value is scaled to whole rows = queries/s)."""
    if rank != 0:
        return None
    import oracle
    w = wl.ALL_WORKLOADS[args.workload]
    d = wl.generate(w)

    def sliced(hs):
        qn = d["q_nope"][:, :hs].contiguous()
        qp = d["q_pe"][:, :hs].contiguous()
        wb = d["wkv_b"].view(128, 256, 512)[:hs].contiguous()
        return lambda row: oracle.mla_sparse_decode(qn, qp, d["kv_cache"], d["pe_cache"], d["end_pos"],
                                                    d["topk_idx"], wb, d["scale"], rows=[row])

    t0 = time.perf_counter()
    sliced(128)(0)
    t_row = max(time.perf_counter() - t0, 1e-4)
    hs = max(1, min(128, int(128 * budget_s / (max(1, args.warmup + args.steps) * t_row))))
    run = sliced(hs)
    times = []
    for it in range(args.warmup + args.steps):
        row = it % w.B
        t0 = time.perf_counter()
        run(row)
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = (hs / 128) * args.steps / total
    sample = (f"each step: {hs} of 128 heads of one batch row (rows rotating), {args.steps} steps, "
              f"{total:.1f} s; a whole row took {t_row:.2f} s")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": w.B, "heads": 128, "S_max": w.S_max, "K": w.K},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # a window of 200 steps (~14 ms); windows repeat until they span 0.5 s
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.ALL_WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the headline decode and its kernels only (no other configurations, projection, "
                         "prefill, end-to-end or CPU baseline): a small footprint for profiler captures")
    ap.add_argument("--sets", type=int, default=0, help="rotating input sets (default: enough to exceed 2x L2)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = reference_arm(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    res, base = gpu_arm(args, rank, world, device)
    if rank == 0:
        if not (args.no_cpu_baseline or args.no_extras):
            res["cpu_baseline"] = cpu_baseline(args, base["host"] if "host" in base else base)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
