#!/usr/bin/env python
"""Decode-step throughput of libhata on synthetic HATA workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one hata_decode_step call over one layer's inputs: encode the
queries, encode + append the new key, Hamming scan with the GQA sum, top-k,
gather + sparse flash-decode.  Steps cycle over R layer buffers whose touched
bytes exceed 4x the L2 size, so every step reads its codes and K/V rows from
HBM.  The K timed steps are CUDA-graph replays bracketed by CUDA events on the
launching stream, with a device synchronize (and a barrier across ranks) on
both sides; the time is the max over ranks.

Prints one JSON line.  --impl reference times the CPU oracle on this host
(rank 0 only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hata_inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "HATA decode-attn steps/s at 32K-128K ctx; achieved HBM GB/s vs peak"
DEFAULT_WORKLOAD = "llama8b_128k"
FALLBACK_HBM_GBS = 6650.0
GRAPH_CHUNK = 1000  # steps per captured graph


# ----------------------------------------------------------------------------
# byte accounting (algorithmic: r/8 per cached token per KV head, 2*k*d*e of
# gathered K/V per KV head, plus q and the output)
# ----------------------------------------------------------------------------

def algorithmic_bytes(wl, seq_lens) -> int:
    e = wl.elem_bytes
    total = 0
    for Lb in seq_lens:
        Lb = int(Lb)
        total += wl.n_kv_heads * (Lb * wl.hash_bits // 8 + 2 * min(wl.k, Lb) * wl.head_dim * e)
    total += 2 * wl.batch * wl.n_q_heads * wl.head_dim * e
    return total


# Sources of the fused kernel: a recorded DRAM traffic figure applies only to them.
KERNEL_SOURCES = ["hata_step.cu", "hata_common.cuh", "hata_ptx.cuh"]


def recorded_traffic(workload_name):
    """DRAM bytes per launch of the fused kernel from the committed ncu record,
    or None when there is no record for this workload or the kernel changed since."""
    rec = os.path.join(ROOT, "profiles", f"fused_step_{workload_name}_traffic.txt")
    if not os.path.exists(rec):
        return None
    fields = {}
    for line in open(rec):
        if line.startswith("#") or ":" not in line:
            continue
        k, v = line.split(":", 1)
        fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "hash_aware_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if fields.get("workload") != workload_name or fields.get("kernel_source_sha256") != h.hexdigest():
        return None
    return int(fields["dram_bytes_per_launch"])


def tensor_peak_bf16():
    """Measured dense bf16 tensor throughput (TFLOP/s, burst) from MEASURED_PEAKS.json, or None."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return None


def peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML, the same counters nvidia-smi reads)
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self.max_mhz = None

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()
            if not self.samples:
                self._sample()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# distributed plumbing (replicas: no data-path collective)
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, dist, device):
    """The largest value over all ranks (the duration of the slowest replica); `dist`
    is torch.distributed when the process group is up, else None (one rank)."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps, seconds):
    """Whole-job steps/s: every replica ran `steps` steps; the job took the slowest one's time."""
    return world * steps / seconds


L2_NOTE = "inputs larger than L2: steps rotate over layer buffers holding more than 4x the L2 size"


def workload_config(wl, seq_lens):
    """The workload's identity, the same in both arms (arm-specific timing details go under "timing")."""
    return {
        "workload": wl.name,
        "batch": wl.batch,
        "n_q_heads": wl.n_q_heads,
        "n_kv_heads": wl.n_kv_heads,
        "head_dim": wl.head_dim,
        "seq_len": int(wl.max_seq) if wl.seq_len_range is None else f"ragged {wl.seq_len_range}",
        "total_cached_tokens": int(np.sum(seq_lens)),
        "hash_bits": wl.hash_bits,
        "top_k": wl.k,
        "kv_dtype": wl.dtype,
        "l2": L2_NOTE,
        "parallelism": "replicas",
    }


# ----------------------------------------------------------------------------
# reference arm: the CPU oracle on this host
# ----------------------------------------------------------------------------

# The oracle's (batch, KV head) units of one decode step are independent, so the
# all-core legs spread them over a process pool.  The pool is forked before any
# CUDA call of this process (a fork after CUDA is initialised is unsafe), and its
# workers read the inputs that the parent made (copy-on-write).
_ORACLE_JOB = None  # (wl, inp, codes) for the pool's workers
_LIMITS = None


def _worker_init():
    global _LIMITS
    from threadpoolctl import threadpool_limits

    _LIMITS = threadpool_limits(1)  # one BLAS thread per worker process


def _oracle_unit(u):
    """One unit of the decode step through the oracle; returns its duration in seconds."""
    import oracle

    wl, inp, codes = _ORACLE_JOB
    b, g = divmod(u % (wl.batch * wl.n_kv_heads), wl.n_kv_heads)
    G = wl.group
    Lb = np.array([int(inp["seq_lens"][b])])
    t0 = time.perf_counter()
    oracle.decode_step(inp["q"][b:b + 1, g * G:(g + 1) * G], inp["K"][b:b + 1, g:g + 1], inp["V"][b:b + 1, g:g + 1],
                       inp["W_H"][g:g + 1], codes[b:b + 1, g:g + 1], Lb, wl.k)
    return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class OraclePool:
    """The CPU oracle over whole decode steps on `cores` worker processes."""

    def __init__(self, wl, inp, cores):
        import multiprocessing

        import oracle

        global _ORACLE_JOB
        codes, _ = oracle.encode_cache(inp["K"], inp["W_H"], inp["seq_lens"])  # the cache before the step
        _ORACLE_JOB = (wl, inp, codes)
        self.units = wl.batch * wl.n_kv_heads
        self.cores = cores
        self.pool = multiprocessing.get_context("fork").Pool(cores, initializer=_worker_init)

    def run_steps(self, n_steps):
        """Wall-clock seconds for n_steps whole steps (all their units queued at once)."""
        t0 = time.perf_counter()
        self.pool.map(_oracle_unit, range(n_steps * self.units), chunksize=1)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(wl, inp, budget_s=12.0):
    """The oracle on this host's cores, before any CUDA call: whole steps over all cores
    (the reported value), plus one thread on a bounded sample of units."""
    from threadpoolctl import threadpool_limits

    cores = host_cores()
    pool = OraclePool(wl, inp, cores)
    try:
        # one thread: units in order until the budget is spent
        elapsed, done = 0.0, 0
        with threadpool_limits(1):
            while done < pool.units and (elapsed < budget_s or done == 0):
                elapsed += _oracle_unit(done)
                done += 1
        single = (done / pool.units) / elapsed
        # all cores: enough whole steps for about budget_s of wall time
        per_unit = elapsed / done
        n_steps = max(1, min(200, math.ceil(budget_s * cores / (per_unit * pool.units))))
        wall = pool.run_steps(n_steps)
    finally:
        pool.close()
    return {
        "value": n_steps / wall,
        "unit": "steps/s",
        "cores": cores,
        "kind": "oracle",
        "sample": f"{n_steps} whole decode steps ({n_steps * pool.units} (batch, KV head) units) over {cores} "
                  "worker processes, one thread each, float64 numpy",
        "single_thread": {"value": single, "unit": "steps/s", "cores": 1,
                          "sample": f"{done} of {pool.units} units of one step, value scaled to whole steps"},
    }


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    inp = make_inputs(wl, seed=args.seed)
    cores = host_cores()
    pool = OraclePool(wl, inp, cores)
    try:
        pool.run_steps(args.warmup)
        wall = pool.run_steps(args.steps)
    finally:
        pool.close()
    value = args.steps / wall
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "steps/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * wall / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, inp["seq_lens"]),
        "timing": {"arm": "CPU oracle, whole decode steps, wall clock",
                   "units_per_step": wl.batch * wl.n_kv_heads, "worker_processes": cores},
        "cpu_baseline": {
            "value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{args.steps} whole decode steps after {args.warmup} warm-up steps, every (batch, KV head) "
                      f"unit queued on {cores} worker processes, one thread each",
        },
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def run_e2e(H, dims, k, steps, layers, stages, in_host, out_host, ws, stream):
    """The end-to-end loop of hash_aware_top_b200/libhata_e2e.so; returns (device ms, host wall ms).

    in_host: pinned [B*Hq + 2*B*Hkv][d] (q, the new K rows, the new V rows); stages: one
    device buffer of that shape per layer; out_host: pinned [B][Hq][d], written by the step."""
    import ctypes

    lib = ctypes.CDLL(os.path.join(os.path.dirname(H.LIB_PATH), "libhata_e2e.so"))
    P = ctypes.c_void_p
    R = len(layers)

    def arr(ts):
        return (P * R)(*[P(t.data_ptr()) for t in ts])

    dms, hms = ctypes.c_float(0), ctypes.c_float(0)
    fn = lib.hata_e2e_run
    fn.restype = ctypes.c_int
    rc = fn(ctypes.byref(dims), int(k), int(steps), R, P(in_host.data_ptr()), P(out_host.data_ptr()), arr(stages),
            arr([lay["K"] for lay in layers]), arr([lay["V"] for lay in layers]), arr([lay["W"] for lay in layers]),
            arr([lay["codes"] for lay in layers]), arr([lay["lens"] for lay in layers]), P(ws.data_ptr()),
            ctypes.c_size_t(ws.numel()), P(stream.cuda_stream), ctypes.byref(dms), ctypes.byref(hms))
    if rc != 0:
        raise RuntimeError(f"end-to-end loop failed: status {rc}")
    return dms.value, hms.value


def e2e_inputs(wl, layer, seq_lens):
    """Pinned host inputs of one end-to-end step -- the layer's queries and the new token's
    K and V rows (those already at slot L_b - 1, so the step's result is unchanged) -- and a
    pinned output buffer."""
    import torch

    rows = lambda C: torch.stack([C[b, :, int(seq_lens[b]) - 1] for b in range(wl.batch)])  # noqa: E731
    flat = torch.cat([layer["q"].reshape(-1, wl.head_dim), rows(layer["K"]).reshape(-1, wl.head_dim),
                      rows(layer["V"]).reshape(-1, wl.head_dim)])
    return flat.cpu().pin_memory(), torch.empty_like(layer["out"], device="cpu").pin_memory()


PREFILL_WORKLOAD = "narrow32_b4_64k"


def tensor_peak_bf16_sustained():
    """Measured dense bf16 tensor throughput held for seconds under the power cap (TFLOP/s), or None."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except (OSError, KeyError, ValueError):
        return None


def bench_prefill_attention(H, dev, local, seed, stream, reps=3, shape=None):
    """Causal prefill attention over the narrow-code workload's prompts (4 x 65,536 tokens,
    32 query / 8 KV heads, r = 32): attention alone, attention with the key encode fused
    (hata_prefill_attention with codes), and the standalone prefill encode of the same keys
    (hata_encode_append), timed interleaved with CUDA events on the launching stream.  The
    attention launches last about 0.3 s, so they run at the clocks the power cap allows; the
    roofline is the sustained measured bf16 peak."""
    import torch

    wl = WORKLOADS[PREFILL_WORKLOAD]
    B, Hq, Hkv, L, r = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.max_seq, wl.hash_bits
    if shape is not None:  # a smaller prompt of the same heads (e.g. for a profiler capture)
        B, L = shape
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 17)
    Q = torch.randn((B, Hq, L, wl.head_dim), device=dev, generator=g).to(torch.bfloat16)
    K = torch.randn((B, Hkv, L, wl.head_dim), device=dev, generator=g).to(torch.bfloat16)
    V = torch.randn((B, Hkv, L, wl.head_dim), device=dev, generator=g).to(torch.bfloat16)
    W = (torch.randn((Hkv, wl.head_dim, r), device=dev, generator=g) / (wl.head_dim ** 0.5)).float()
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    out = torch.empty_like(Q)
    codes = torch.zeros((B, Hkv, L, wl.words), dtype=torch.int32, device=dev)
    d = H.dims_for(B, Hq, Hkv, wl.head_dim, r, L, "bf16")
    ws = torch.zeros(H.hata_prefill_workspace_size(d), dtype=torch.uint8, device=dev)
    ews = torch.zeros(H.hata_workspace_size(d, wl.k), dtype=torch.uint8, device=dev)
    calls = {
        "attention": lambda: H.hata_prefill_attention(d, Q, K, V, None, None, lens, 0.0, out, ws, stream),
        "fused": lambda: H.hata_prefill_attention(d, Q, K, V, W, codes, lens, 0.0, out, ws, stream),
        "encode": lambda: H.hata_encode_append(d, K, Hkv, L, L, lens, W, codes, L, ews, stream),
    }
    times = {n: [] for n in calls}
    with torch.cuda.stream(stream):
        for fn in calls.values():
            fn()
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            for _ in range(reps):
                for name, fn in calls.items():
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                    e1.synchronize()
                    times[name].append(e0.elapsed_time(e1))
    for w_ in (ws, ews):
        if H.hata_read_device_status(w_) != 0:
            raise RuntimeError("device status set by the prefill attention or encode")
    ms = {n: statistics.median(v) for n, v in times.items()}
    flops = 4.0 * wl.head_dim * Hq * B * L * (L + 1) / 2  # q.K and P.V over the causal triangle
    tflops = flops / (ms["attention"] * 1e-3) / 1e12
    name = PREFILL_WORKLOAD if shape is None else f"{PREFILL_WORKLOAD} heads"
    res = {"workload": f"{name}: {B} x {L}-token prompts, {Hq}/{Hkv} heads, d {wl.head_dim}, r {r}, bf16",
           "kernel": "hata_prefill_attention (tcgen05 causal attention; key encode fused on the diagonal tile)",
           "reps": reps, "attention_ms": ms["attention"], "fused_ms": ms["fused"],
           "fused_encode_overhead_ms": ms["fused"] - ms["attention"],
           "standalone_encode_ms": ms["encode"], "flops": flops, "tflops": tflops,
           "clocks": clk.summary()}
    tpeak = tensor_peak_bf16_sustained()
    if tpeak:
        res["peak_tflops"] = tpeak
        res["peak_kind"] = "measured sustained"
        res["frac_of_tensor_peak"] = tflops / tpeak
    del Q, K, V, out, codes
    torch.cuda.empty_cache()
    return res


def graph_upload(g, stream):
    """Upload an instantiated graph to the device before it is timed, so that the first
    timed replay does not pay for it (driver call cuGraphUpload on the graph's exec handle)."""
    import ctypes

    try:
        cuda = ctypes.CDLL("libcuda.so.1")
        cuda.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        rc = cuda.cuGraphUpload(ctypes.c_void_p(int(g.raw_cuda_graph_exec())), ctypes.c_void_p(stream.cuda_stream))
        return rc == 0
    except (OSError, AttributeError, RuntimeError):
        return False


WARM_MIN_S = 0.05  # the warm-up runs for at least this long (whole rotations of the layer buffers)


def warmup_pass_steps(warmup, rotation):
    """Steps in one replay of the warm-up graph: at least `warmup` (and at least one), rounded
    up to whole rotations over the `rotation` layer buffers."""
    rotation = max(1, rotation)
    return -(-max(warmup, 1) // rotation) * rotation


def graph_time(step, steps, warmup, stream, dist=None, sampler=None, rotation=1):
    """Milliseconds for `steps` calls of step(i) replayed from CUDA graphs, after the
    warm-up: CUDA events on the launching stream, a synchronize (and a barrier across
    ranks) on both sides.

    The warm-up is at least `warmup` steps, in whole rotations over the `rotation` layer
    buffers that step(i) cycles through, replayed until WARM_MIN_S has passed, so that the
    timed steps start from the steady state of a running decode loop that keeps cycling
    over all its layers (a cold rotation measured 20.4 us/step over 20 steps at 128K,
    against 19.3 after this warm-up and 18.9 over 2000 steps).  The number of warm-up
    steps run is left in graph_time.last_warmup_steps."""
    import contextlib

    import torch

    def capture(n, events=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if events:
                events[0].record(stream)
            for i in range(n):
                step(i)
            if events:
                events[1].record(stream)
        return g

    with torch.cuda.stream(stream):
        for i in range(3):  # eager calls before capture (first-launch setup)
            step(i)
    torch.cuda.synchronize()
    chunk = min(steps, GRAPH_CHUNK)
    # A run that fits one graph records its timing events inside it (event-record nodes), so
    # they bracket exactly the timed steps on the device and not the host's submission of
    # the graph; longer runs record them around the replays (the submission gap is then
    # spread over GRAPH_CHUNK steps per graph).
    ev0, ev1 = torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)
    inside = steps <= GRAPH_CHUNK
    g_chunk = capture(chunk, (ev0, ev1) if inside else None)
    rem = steps % chunk
    g_rem = capture(rem) if rem else None
    n_warm = warmup_pass_steps(warmup, rotation)
    g_warm = capture(n_warm)
    for g in (g_chunk, g_rem, g_warm):
        if g is not None:
            graph_upload(g, stream)
    torch.cuda.synchronize()
    reps = 0
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):  # graph replays go to torch's current stream: the timed one
        while True:
            g_warm.replay()
            torch.cuda.synchronize()
            reps += 1
            if time.perf_counter() - t0 >= WARM_MIN_S:
                break
    graph_time.last_warmup_steps = reps * n_warm  # this rank's; the barrier below aligns the ranks
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with (sampler or contextlib.nullcontext()), torch.cuda.stream(stream):
        if not inside:
            ev0.record(stream)
        for _ in range(steps // chunk):
            g_chunk.replay()
        if g_rem is not None:
            g_rem.replay()
        if not inside:
            ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    if ms / steps < 1e-4:
        raise RuntimeError(f"implausible step time {ms / steps * 1e3:.3f} us")
    del g_chunk, g_rem, g_warm
    return ms


class LayerSet:
    """R copies ("layers") of one workload's device buffers, so that consecutive steps read
    different memory and the bytes touched per rotation exceed 4x the L2 size."""

    def __init__(self, H, wl, inp, dev, layers=None):
        import torch

        self.wl, self.inp = wl, inp
        self.tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.dims = H.dims_for(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.hash_bits, wl.max_seq,
                               wl.dtype)
        self.step_bytes = algorithmic_bytes(wl, inp["seq_lens"])
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.R = max(2, math.ceil(4 * l2 / self.step_bytes)) if layers is None else layers
        self.l2 = l2

        def to_dev(a):
            return torch.from_numpy(a).to(dev).to(self.tdt)

        base = {"q": to_dev(inp["q"]), "K": to_dev(inp["K"]), "V": to_dev(inp["V"]),
                "W": torch.from_numpy(inp["W_H"]).to(dev), "lens": torch.from_numpy(inp["seq_lens"]).to(dev)}
        self.ws = torch.empty(H.hata_workspace_size(self.dims, wl.k), dtype=torch.uint8, device=dev)
        H.hata_workspace_init(self.ws)
        # prefill: encode every cached key through the library
        codes0 = torch.zeros((wl.batch, wl.n_kv_heads, wl.max_seq, wl.words), dtype=torch.int32, device=dev)
        H.hata_encode_append(self.dims, base["K"], wl.n_kv_heads, wl.max_seq, wl.max_seq, base["lens"], base["W"],
                             codes0, wl.max_seq, self.ws)
        self.layers = []
        for i in range(self.R):
            lay = {n: (t if i == 0 else t.clone()) for n, t in base.items()}
            lay["codes"] = codes0 if i == 0 else codes0.clone()
            lay["out"] = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=self.tdt, device=dev)
            self.layers.append(lay)
        torch.cuda.synchronize()

    def timing_note(self, steps=None):
        note = {"layer_buffers": self.R, "mb_touched_per_rotation": round(self.R * self.step_bytes / 1e6),
                "l2_mb": round(self.l2 / 1e6)}
        if steps is not None:
            note["events"] = ("recorded inside the one CUDA graph of the timed steps" if steps <= GRAPH_CHUNK else
                              f"recorded around the replays of CUDA graphs of {GRAPH_CHUNK} steps")
        return note


def time_prefill_encode(H, ls, stream):
    """hata_encode_append over every cached key of the layer buffers (prefill form), timed with CUDA
    events on the launching stream; the keys/s, bytes and tensor-core figures of one call."""
    import torch

    wl, layers, R, inp = ls.wl, ls.layers, ls.R, ls.inp
    reps = max(2, min(R, 8))
    with torch.cuda.stream(stream):
        L0 = layers[0]
        H.hata_encode_append(ls.dims, L0["K"], wl.n_kv_heads, wl.max_seq, wl.max_seq, L0["lens"], L0["W"],
                             L0["codes"], wl.max_seq, ls.ws, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            L = layers[i % R]
            H.hata_encode_append(ls.dims, L["K"], wl.n_kv_heads, wl.max_seq, wl.max_seq, L["lens"], L["W"],
                                 L["codes"], wl.max_seq, ls.ws, stream)
        e1.record(stream)
        e1.synchronize()
    pre_ms = e0.elapsed_time(e1) / reps
    n_keys = int(sum(int(Lb) for Lb in inp["seq_lens"])) * wl.n_kv_heads
    pre_bytes = n_keys * (wl.head_dim * (2 if wl.dtype == "bf16" else 4) + max(wl.hash_bits // 8, 2))
    res = {"kernel": "hata_encode_append (prefill form; bf16 keys: tcgen05 tensor cores)",
           "us_per_call": pre_ms * 1e3, "keys": n_keys,
           "keys_per_s": n_keys / (pre_ms * 1e-3), "bytes_per_call": pre_bytes,
           "achieved_gbs": pre_bytes / (pre_ms * 1e-3) / 1e9,
           "tflops": 2.0 * n_keys * wl.head_dim * wl.hash_bits / (pre_ms * 1e-3) / 1e12}
    if wl.dtype == "bf16" and 32 <= wl.hash_bits <= 128:
        # the tensor cores run W_H as three bf16 parts: 3x the algorithmic flops
        res["mma_tflops"] = 3.0 * res["tflops"]
        tpeak = tensor_peak_bf16()
        if tpeak:
            res["frac_of_tensor_peak"] = res["mma_tflops"] / tpeak
    if H.hata_read_device_status(ls.ws) != 0:
        raise RuntimeError("device status set by the prefill encode")
    peak, _ = peak_hbm()
    res["frac_of_peak"] = res["achieved_gbs"] / peak
    return res


def run_gpu(args, wl):
    world, rank, local = dist_env()
    inp = make_inputs(wl, seed=args.seed)
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, inp)  # before the first CUDA call of this process (forked pool)

    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import hash_aware_top_b200 as H

    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    ls = LayerSet(H, wl, inp, dev, args.layers)
    dims, R, layers, ws, step_bytes = ls.dims, ls.R, ls.layers, ls.ws, ls.step_bytes

    def step(i):
        L = layers[i % R]
        H.hata_decode_step(dims, L["q"], L["K"], L["V"], L["W"], L["codes"], L["lens"], wl.k, 0.0, L["out"], None,
                           None, ws, stream)

    sampler = ClockSampler(local)
    ms = graph_time(step, args.steps, args.warmup, stream, dist, sampler, rotation=R)
    warm_run = graph_time.last_warmup_steps
    ms = max_over_ranks(ms, dist, dev)
    if dist:
        dist.barrier()
    status = H.hata_read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status}: {H.hata_status_string(status)}")
    ms_per_step = ms / args.steps
    value = job_throughput(world, args.steps, ms / 1e3)
    # end to end through the public C ABI (a native loop, hash_aware_top_b200/e2e): every step
    # copies its inputs (q and the new token's K and V rows) from pinned host memory in one
    # copy, appends the rows to the caches (hata_append_kv), runs hata_decode_step with the
    # output in pinned host memory, and waits for it
    # (at least 1000 timed steps, after untimed loop calls for at least WARM_MIN_S, so that a
    # short run's figure is the running loop's and not its cold start's)
    e2e_steps = max(1000, min(args.steps, 2000))
    in_host, out_host = e2e_inputs(wl, layers[0], inp["seq_lens"])
    stages = [torch.empty_like(in_host, device=dev) for _ in layers]
    h2d = in_host.numel() * in_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    e2e_warm, t_w = 0, time.perf_counter()
    while e2e_warm == 0 or time.perf_counter() - t_w < WARM_MIN_S:  # warm-up
        run_e2e(H, dims, wl.k, 100, layers, stages, in_host, out_host, ws, stream)
        e2e_warm += 100
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e2e_dev_ms, e2e_host_ms = run_e2e(H, dims, wl.k, e2e_steps, layers, stages, in_host, out_host, ws, stream)
    e2e_s = max_over_ranks(e2e_dev_ms / 1e3, dist, dev)
    e2e_value = job_throughput(world, e2e_steps, e2e_s)

    # the dense flash-decode baseline on the same layer buffers (the comparison the pages report)
    dense = None
    if wl.dtype == "bf16" and wl.n_q_heads // wl.n_kv_heads <= 8:
        dws = torch.zeros(H.hata_dense_workspace_size(dims), dtype=torch.uint8, device=dev)

        def dense_step(i):
            L = layers[i % R]
            H.hata_dense_decode(dims, L["q"], L["K"], L["V"], L["lens"], 0.0, L["out"], dws, stream)

        d_steps = min(args.steps, 2000)
        d_ms = graph_time(dense_step, d_steps, args.warmup, stream, rotation=R) / d_steps
        d_bytes = sum(2 * int(Lb) * wl.n_kv_heads * wl.head_dim * 2 for Lb in inp["seq_lens"]) + \
            2 * wl.batch * wl.n_q_heads * wl.head_dim * 2
        dense = {"kernel": "hata_dense_decode (dense flash-decode, bf16 tensor-core tiles)", "steps": d_steps,
                 "us_per_step": d_ms * 1e3, "bytes_per_step": d_bytes,
                 "achieved_gbs": d_bytes / (d_ms * 1e-3) / 1e9,
                 "hata_speedup": d_ms / ms_per_step}

    # prefill encode (hata_encode_append over every cached key of every layer buffer)
    prefill = time_prefill_encode(H, ls, stream)

    # the same step over a paged cache: every layer's K, V and codes are rearranged in
    # place into pools of 256-token blocks placed by a random (non-contiguous) block
    # table, so the paged step reads the same data and selects the same rows
    paged = None
    bs_p = 256
    if wl.max_seq % bs_p == 0 and H.hata_decode_step_kernel_count(dims, wl.k) >= 1:
        max_blocks = wl.max_seq // bs_p
        n_blocks = wl.batch * max_blocks
        gen = torch.Generator().manual_seed(args.seed + 1)
        perm = torch.randperm(n_blocks, generator=gen)
        btab = perm.to(torch.int32).reshape(wl.batch, max_blocks).to(dev)
        pool = (n_blocks, wl.n_kv_heads, bs_p)
        where = perm.to(dev)

        def to_pool(t):  # [B][Hkv][Lmax][X] -> pool blocks, in place
            X = t.shape[-1]
            blocks = t.view(wl.batch, wl.n_kv_heads, max_blocks, bs_p, X).permute(0, 2, 1, 3, 4).reshape(
                n_blocks, wl.n_kv_heads, bs_p, X)
            out = torch.empty(blocks.shape, dtype=blocks.dtype, device=blocks.device)
            out[where] = blocks
            t.view(-1).copy_(out.view(-1))

        for L in layers:
            for name in ("K", "V", "codes"):
                to_pool(L[name])
        torch.cuda.synchronize()

        def paged_step(i):
            L = layers[i % R]
            H.hata_decode_step_paged(dims, L["q"], L["K"].view(*pool, wl.head_dim), L["V"].view(*pool, wl.head_dim),
                                     L["W"], L["W"], L["codes"].view(*pool, wl.words), btab, bs_p, L["lens"], wl.k,
                                     0.0, L["out"], None, None, ws, stream)

        p_steps = min(args.steps, 2000)
        p_ms = graph_time(paged_step, p_steps, args.warmup, stream, rotation=R) / p_steps
        paged = {"kernel": "hata_decode_step_paged (256-token blocks, random block table)", "steps": p_steps,
                 "us_per_step": p_ms * 1e3, "achieved_gbs": step_bytes / (p_ms * 1e-3) / 1e9,
                 "vs_unpaged": ms_per_step / p_ms}
    timing = ls.timing_note(args.steps)
    timing["warmup_steps_run"] = warm_run  # >= args.warmup: whole rotations for at least WARM_MIN_S
    del ls, layers
    torch.cuda.empty_cache()

    peak, peak_kind = peak_hbm()
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    if dense is not None:
        dense["frac_of_peak"] = dense["achieved_gbs"] / peak

    # the other context lengths the metric names (32K-128K): the same step, timed the same way
    workloads = {}
    for name in (args.also or []):
        if name == wl.name:
            continue
        wl2 = WORKLOADS[name]
        ls2 = LayerSet(H, wl2, make_inputs(wl2, seed=args.seed), dev)

        def step2(i, ls2=ls2):
            L = ls2.layers[i % ls2.R]
            H.hata_decode_step(ls2.dims, L["q"], L["K"], L["V"], L["W"], L["codes"], L["lens"], wl2.k, 0.0,
                               L["out"], None, None, ls2.ws, stream)

        n2 = min(args.steps, 2000)
        ms2 = graph_time(step2, n2, args.warmup, stream, rotation=ls2.R) / n2
        if H.hata_read_device_status(ls2.ws) != 0:
            raise RuntimeError(f"device status set on workload {name}")
        gbs2 = ls2.step_bytes / (ms2 * 1e-3) / 1e9
        workloads[name] = {"steps": n2, "us_per_step": ms2 * 1e3, "steps_per_s": 1e3 / ms2,
                           "algorithmic_bytes_per_step": ls2.step_bytes, "achieved_gbs": gbs2,
                           "frac": gbs2 / peak, **ls2.timing_note(n2),
                           "prefill_encode": time_prefill_encode(H, ls2, stream)}
        del ls2
        torch.cuda.empty_cache()

    prefill_attn = None
    if not args.no_prefill_attention:
        prefill_attn = bench_prefill_attention(H, dev, local, args.seed, stream, shape=args.prefill_shape)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic",
        "config": workload_config(wl, inp["seq_lens"]),
        "timing": timing,
        "roofline": {
            "bound": "hbm",
            "kernel": "hata_decode_step (whole step)",
            "achieved": achieved,
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": recorded_traffic(wl.name),
            "algorithmic_bytes_per_step": step_bytes,
        },
        "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "warmup_steps_run": e2e_warm, "host_wall_ms": e2e_host_ms,
                "loop": "native loop over the C ABI, every step: one H2D of q and the new K/V rows, "
                        "hata_append_kv, hata_decode_step writing its output into mapped pinned host memory "
                        "(the D2H bytes), stream synchronize"},
        "gpu_launches": args.steps * H.hata_decode_step_kernel_count(dims, wl.k),
        "workloads": workloads,
        "dense_baseline": dense,
        "paged_step": paged,
        "prefill_encode": prefill,
        "prefill_attention": prefill_attn,
        "clocks": sampler.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="hata", choices=["hata", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=None, help="layer buffers to rotate over (default: > 4x L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill-attention", action="store_true",
                    help="skip the prefill attention timing (about 3 s of GPU time)")
    ap.add_argument("--prefill-shape", type=int, nargs=2, metavar=("B", "L"), default=None,
                    help="prompts of the prefill attention leg (default: the narrow-code workload's 4 x 65536)")
    ap.add_argument("--also", nargs="*", default=None,
                    help="other workloads timed in the same run (default: llama8b_32k beside the 128K headline)")
    args = ap.parse_args(argv)
    if args.also is None:
        args.also = ["llama8b_32k"] if args.workload == "llama8b_128k" else []
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
