#!/usr/bin/env python
"""Benchmark of the fused KV-cache rotate-and-quantize path on B200.

One step = one pass of the whole path over one batch: kvq_quantize of the
batch (fp16 -> int4 codes + fp16 group scales) followed by kvq_dequantize of
the result (-> fp16).  The default batch is a Qwen3-8B-shaped prefill cache:
36 layers x 8 KV heads x 32768 tokens x (K, V) = 18,874,368 vectors of D=128,
group 32, synthetic Student-t(3) values with 4 outlier channels x20.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torchrun, one process per GPU; every rank quantises its own
cache shard of the same shape (weak scaling, no collective on the data path);
the time is the maximum over ranks.  Rank 0 prints one JSON line.

`value` (Gvec/s, higher is better) = vectors of all ranks / device time of
the K timed steps, inputs resident in HBM.  `e2e` is the same metric through
the public API with the inputs in pinned host memory: each step copies the
fp16 batch host->device, quantises, dequantises and copies the fp16 result
back, chunked over three streams so that the copies overlap.  `roofline`
reports the slower kernel's algorithmic HBM bytes per launch over its
CUDA-event duration against the measured copy bandwidth.  `cpu_baseline` is
the CPU oracle timed on the host's cores over a bounded sample of the same
workload.  `--impl reference` times that oracle alone as the reference arm.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_quantization_02_b200 import workloads  # noqa: E402

METRIC = "Gvec/s quantize+pack and dequant at D=128; achieved HBM GB/s vs B200 peak"
UNIT = "Gvec/s"
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "kvq_traffic_slices.json")


def bytes_per_vector(D: int, G: int) -> int:
    """Algorithmic HBM bytes per vector, the same for quantize and dequant:
    2D (fp16 row) + D/2 (codes) + 2D/G (fp16 scales)."""
    return 2 * D + D // 2 + 2 * (D // G)


# ---------------------------------------------------------------------------
# distributed plumbing (host logic, covered by the gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def shard_seed_offset(rank: int) -> int:
    """Each rank draws a different cache shard of the same shape."""
    return 1000 + rank


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread; read-only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - report, do not fail the bench
            self._nv = None
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception as e:  # noqa: BLE001
                self.error = repr(e)
                return
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit]
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": names,
               "samples": len(self.samples), "source": "NVML, polled during the timed region"}
        if self.error:
            out["error"] = self.error
        return out


# ---------------------------------------------------------------------------
# peaks and the committed ncu traffic summary
# ---------------------------------------------------------------------------

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def traffic_per_launch(kernel: str, units: int):
    """DRAM bytes per launch from the committed ncu summary, scaled by the
    units one launch processes (vectors, or cache rows for the attention), or
    None when that kernel's source changed since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except Exception:  # noqa: BLE001
        return None
    k = t.get("kernels", {}).get(kernel)
    if not k:
        return None
    src = os.path.join(ROOT, k.get("source", ""))
    if not os.path.isfile(src) or k.get("source_sha256") != source_sha(src):
        return None
    return k["dram_bytes_per_unit"] * units


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample, all host cores via threads; ctypes
# releases the GIL during each call)
# ---------------------------------------------------------------------------

class OracleTimer:
    """Times the CPU oracle (quantize + dequantize) over a bounded sample of a
    workload, split across host threads.  The sample is drawn once (a pool of
    at most 2^18 rows, tiled to the sample size: the oracle's work per row
    does not depend on the values)."""

    def __init__(self, w: workloads.Workload, G: int, target_s: float,
                 threads: int | None = None):
        import numpy as np
        import oracle

        self.o = oracle.get()
        self.G = G
        self.lam, self.s = workloads.params(w.D, w.seed)
        self.threads = threads or len(os.sched_getaffinity(0))
        probe = workloads.host_rows(w, 2048, seed_offset=77)
        t0 = time.perf_counter()
        self._one(probe)
        per_row = (time.perf_counter() - t0) / len(probe)
        rows = int(target_s * self.threads / max(per_row, 1e-9))
        self.rows = max(self.threads * 256, min(rows, 1 << 22))
        pool = workloads.host_rows(w, min(self.rows, 1 << 18), seed_offset=78)
        reps = -(-self.rows // len(pool))
        x16 = np.concatenate([pool] * reps)[: self.rows]
        self.parts = [np.ascontiguousarray(p) for p in np.array_split(x16, self.threads)]

    def set_rows(self, n: int, w: workloads.Workload):
        """Time exactly the n rows of workload w (drawn on the host)."""
        import numpy as np
        x16 = workloads.host_rows(w, n, seed_offset=79)
        self.rows = n
        self.parts = [np.ascontiguousarray(p) for p in np.array_split(x16, self.threads) if len(p)]

    def _one(self, x16):
        packed, scales = self.o.quantize(x16, self.lam, self.s, self.G)
        self.o.dequantize(packed, scales, self.lam, self.s, self.G)

    def run(self) -> float:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(self.threads) as ex:
            t0 = time.perf_counter()
            list(ex.map(self._one, self.parts))
            return time.perf_counter() - t0


def oracle_extra_timings(w, G, target_s):
    """The oracle on one thread (a bounded sample of the same workload, a
    tenth of the time budget), and the three smaller configurations timed in
    full on all host threads: tiny (256 vectors), qwen2.5-1.5b (458,752) and
    gemma-3-1b (212,992, D = 256, G = 32 and 64)."""
    one = OracleTimer(w, G, max(target_s / 10.0, 0.5), threads=1)
    dt1 = one.run()
    res = {"single_thread": {"value": one.rows / dt1 / 1e9, "unit": UNIT,
                             "sample": f"{one.rows} vectors, {dt1:.2f} s on 1 thread"}}
    full = {}
    for name, groups in (("tiny", None), ("qwen2.5-1.5b", None), ("gemma-3-1b", (32, 64))):
        c = workloads.WORKLOADS[name]
        for g in groups or (c.groups[0],):
            ot = OracleTimer(c, g, 0.0)
            ot.set_rows(c.n_vec, c)
            dt = ot.run()
            full[f"{name}_g{g}"] = {"vectors": c.n_vec, "seconds": round(dt, 4),
                                    "gvec_s": c.n_vec / dt / 1e9, "threads": ot.threads}
    res["configs_full"] = full
    return res


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args):
    import torch
    from kv_cache_quantization_02_b200 import kvq

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    w = workloads.WORKLOADS[args.workload]
    G = args.group or w.groups[0]
    n = args.n_vec or w.n_vec
    D = w.D
    lam, s = workloads.params(D, w.seed)
    lam_t = torch.from_numpy(lam).to(dev)
    s_t = torch.from_numpy(s).to(dev)

    x = workloads.device_rows(w, n, dev, seed_offset=shard_seed_offset(rank))
    packed = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
    out = torch.empty((n, D), dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kvq.quantize(x, lam_t, s_t, G, packed=packed, scales=scales, stream=stream)
        kvq.dequantize(packed, scales, lam_t, s_t, G, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            kvq.quantize(x, lam_t, s_t, G, packed=packed, scales=scales, stream=stream)
            ev[i][1].record(stream)
            kvq.dequantize(packed, scales, lam_t, s_t, G, out=out, stream=stream)
            ev[i][2].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    elapsed_ms = start.elapsed_time(end)
    q_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    d_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    q_ms = max_over_ranks(q_ms, world, dev)
    d_ms = max_over_ranks(d_ms, world, dev)

    extra = {}
    if args.variants_only:
        extra = {"codec_variants": run_variants(torch, kvq, dev, stream, x, out, s_t, G, w)}
        if w.D == 128:
            extra["srft_lengths"] = run_srft_lengths(torch, kvq, dev, stream)
    elif args.attention_only:
        cache = build_decode_cache(torch, kvq, dev, stream, lam_t, s_t, G, args.attn_seqs)
        extra = {"attention_decode": run_attention(torch, kvq, dev, stream, lam_t, s_t, G, cache)}
        del cache
        torch.cuda.empty_cache()
        extra["attention_decode_paper_format"] = run_attention_paper_format(torch, kvq, dev, stream,
                                                                            args.attn_seqs)
        extra["attention_decode_gemma"] = run_attention_gemma(torch, kvq, dev, stream, args.attn_seqs)
    elif args.configs_only:
        extra = {"configs": run_configs(torch, kvq, dev, stream)}
    elif args.tc_only:
        extra = {"dequantize_tensor_cores": run_dequant_tc(torch, kvq, dev, stream, x, out, lam_t, s_t)}
    elif args.roundtrip_only:
        rt_ms = _event_ms(torch, stream,
                          lambda: kvq.roundtrip(x, lam_t, s_t, G, out=out, stream=stream), 10)
        extra = {"roundtrip_ms": round(rt_ms, 5)}
    elif not args.no_extra:
        extra = run_extras(torch, kvq, dev, stream, x, out, lam_t, s_t, G, w, args.attn_seqs)

    bpv = bytes_per_vector(D, G)
    total_vec = n * world
    value = total_vec * K / (elapsed_ms / 1e3) / 1e9
    peak, peak_kind = hbm_peak()
    kern = {"kvq_quantize": q_ms, "kvq_dequantize": d_ms}
    top = max(kern, key=kern.get)
    achieved = bpv * n / (kern[top] / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, torch, kvq, dev, x, lam_t, s_t, G, world)
    del x, out, packed, scales
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        ot = OracleTimer(w, G, args.cpu_seconds)
        dt = ot.run()
        cpu = {"value": ot.rows / dt / 1e9, "unit": UNIT, "cores": ot.threads,
               "kind": "oracle",
               "sample": f"{ot.rows} vectors of the {w.name} distribution (host-drawn), "
                         f"quantize+dequantize, {dt:.1f} s on {ot.threads} threads",
               **oracle_extra_timings(w, G, args.cpu_seconds)}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(elapsed_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": w.name, "n_vec_per_gpu": n, "D": D, "group": G, "shape": w.shape,
            "values": w.note, "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"weak: {world} independent cache shard(s), no collective",
            "global_batch": total_vec,
        },
        "detail": {
            "quantize_ms": round(q_ms, 5), "dequantize_ms": round(d_ms, 5),
            "quantize_gvec_s": round(n * world / (q_ms / 1e3) / 1e9, 4),
            "dequantize_gvec_s": round(n * world / (d_ms / 1e3) / 1e9, 4),
            "quantize_gbs": round(bpv * n / (q_ms / 1e3) / 1e9, 1),
            "dequantize_gbs": round(bpv * n / (d_ms / 1e3) / 1e9, 1),
            "bytes_per_vector": bpv,
            "frac_of_8tbs": {"kvq_quantize": round(bpv * n / (q_ms / 1e3) / 1e9 / 8000, 4),
                             "kvq_dequantize": round(bpv * n / (d_ms / 1e3) / 1e9 / 8000, 4)},
            **extra,
        },
        "roofline": {
            "kernel": top, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": traffic_per_launch(top, n),
            "algorithmic_bytes_per_launch": bpv * n,
        },
        "gpu_launches": 2 * K * world,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    return line


def _event_ms(torch, stream, fn, reps):
    fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record(stream)
    for i in range(reps):
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    t = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(reps))
    return t[len(t) // 2]


def run_extras(torch, kvq, dev, stream, x, out, lam_t, s_t, G, w, attn_seqs=64):
    """Secondary figures, outside the timed steps: the fused round trip on the
    same batch, and the decode-time append of one new K and V token for 64
    sequences x 36 layers x 8 KV heads into their rows of a cache."""
    n, D = x.shape
    rt_ms = _event_ms(torch, stream,
                      lambda: kvq.roundtrip(x, lam_t, s_t, G, out=out, stream=stream), 10)
    a = workloads.WORKLOADS["decode-append"]
    na = a.n_vec
    T = 64                                        # cache slots per (sequence, layer, head)
    xa = workloads.device_rows(a, na, dev)
    idx = torch.arange(na, device=dev, dtype=torch.int64) * T + (T - 1)
    cpk = torch.empty((na * T, D // 2), dtype=torch.uint8, device=dev)
    csc = torch.empty((na * T, D // G), dtype=torch.float16, device=dev)
    ap_ms = _event_ms(torch, stream, lambda: kvq.quantize_rows(
        xa, lam_t, s_t, G, idx, cpk, csc, stream=stream), 50)
    del xa, cpk, csc
    res = {
        "roundtrip_ms": round(rt_ms, 5),
        "roundtrip_gbs": round(n * 4 * D / (rt_ms / 1e3) / 1e9, 1),
        "decode_append_vectors": na,
        "decode_append_us": round(ap_ms * 1e3, 2),
        "decode_append_gvec_s": round(na / (ap_ms / 1e3) / 1e9, 3),
    }
    if D == 128:
        res["codec_variants"] = run_variants(torch, kvq, dev, stream, x, out, s_t, G, w)
        res["dequantize_tensor_cores"] = run_dequant_tc(torch, kvq, dev, stream, x, out, lam_t, s_t)
        res["srft_lengths"] = run_srft_lengths(torch, kvq, dev, stream)
        cache = build_decode_cache(torch, kvq, dev, stream, lam_t, s_t, G, attn_seqs)
        res["attention_decode"] = run_attention(torch, kvq, dev, stream, lam_t, s_t, G, cache)
        res["decode_step"] = run_decode_step(torch, kvq, dev, stream, lam_t, s_t, G, cache,
                                             steps=1000 if attn_seqs == 64 else 20)
        del cache
        torch.cuda.empty_cache()
        res["attention_decode_paper_format"] = run_attention_paper_format(torch, kvq, dev, stream, attn_seqs)
        res["attention_decode_gemma"] = run_attention_gemma(torch, kvq, dev, stream, attn_seqs)
        res["configs"] = run_configs(torch, kvq, dev, stream)
        res["d256"] = run_d256(torch, kvq, dev, stream)
    # last, so that its seconds under the power cap do not slow the figures above
    res["sustained"] = run_sustained(torch, kvq, dev, stream, x, out, lam_t, s_t, G)
    return res


def _flushed_ms(torch, stream, fn, reps, flush, clean=None):
    """Per-rep CUDA-event times of fn, the L2 flushed before each rep by a
    write of `flush` (twice the L2's 126 MB); with `clean` (another buffer
    larger than L2), a read of it follows the write, so the L2 holds clean
    lines and the timed kernel does not pay for writing back the flush's
    dirty ones.  (median, min, max) in ms."""
    fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        if clean is not None:
            clean.max()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) for a, b in ev)
    return t[len(t) // 2], t[0], t[-1]


CONFIG_CASES = (("tiny", 32), ("qwen2.5-1.5b", 32), ("gemma-3-1b", 32), ("gemma-3-1b", 64))


def run_configs(torch, kvq, dev, stream, reps=20):
    """The smaller configurations (each batch fits in L2): quantize and
    dequantize timed one rep at a time with the L2 flushed before each rep;
    median, min and max in microseconds.  A second pair of figures reads a
    second 256 MB buffer after the flush's write: the write leaves up to the
    L2's 126 MB of dirty lines, whose write-back the timed kernel otherwise
    pays (comparable to these batches' own bytes)."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clean = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    peak, _ = hbm_peak()
    res = {"protocol": f"{reps} reps, L2 flushed (256 MB write) before each; median/min/max; "
                       "*_clean: the write followed by a 256 MB read"}
    for name, G in CONFIG_CASES:
        w = workloads.WORKLOADS[name]
        D, n = w.D, w.n_vec
        lam, s = workloads.params(D, w.seed)
        lt, st = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
        x = workloads.device_rows(w, n, dev)
        pk = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty((n, D // G), dtype=torch.float16, device=dev)
        out = torch.empty_like(x)
        q = _flushed_ms(torch, stream, lambda: kvq.quantize(
            x, lt, st, G, packed=pk, scales=sc, stream=stream), reps, flush)
        d = _flushed_ms(torch, stream, lambda: kvq.dequantize(
            pk, sc, lt, st, G, out=out, stream=stream), reps, flush)
        qc = _flushed_ms(torch, stream, lambda: kvq.quantize(
            x, lt, st, G, packed=pk, scales=sc, stream=stream), reps, flush, clean)
        dc = _flushed_ms(torch, stream, lambda: kvq.dequantize(
            pk, sc, lt, st, G, out=out, stream=stream), reps, flush, clean)
        bpv = bytes_per_vector(D, G)
        res[f"{name}_g{G}"] = {
            "n_vec": n, "D": D, "G": G, "bytes_per_vector": bpv,
            "quantize_us": [round(v * 1e3, 2) for v in q],
            "dequantize_us": [round(v * 1e3, 2) for v in d],
            "quantize_gvec_s": round(n / (q[0] / 1e3) / 1e9, 3),
            "dequantize_gvec_s": round(n / (d[0] / 1e3) / 1e9, 3),
            "quantize_gbs": round(bpv * n / (q[0] / 1e3) / 1e9, 1),
            "dequantize_gbs": round(bpv * n / (d[0] / 1e3) / 1e9, 1),
            "quantize_us_clean": [round(v * 1e3, 2) for v in qc],
            "dequantize_us_clean": [round(v * 1e3, 2) for v in dc],
            "quantize_gbs_clean": round(bpv * n / (qc[0] / 1e3) / 1e9, 1),
            "dequantize_gbs_clean": round(bpv * n / (dc[0] / 1e3) / 1e9, 1),
        }
        del x, pk, sc, out
    del flush, clean
    torch.cuda.empty_cache()
    return res


def run_d256(torch, kvq, dev, stream, n=9_437_184):
    """D = 256 on a batch as large in bytes as the prefill batch: 9,437,184
    rows of the Gemma-3-1B distribution (6.19 GB per launch at G = 32), far
    above L2; G = 32 and 64."""
    w = workloads.WORKLOADS["gemma-3-1b"]
    D = w.D
    lam, s = workloads.params(D, w.seed)
    lt, st = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
    x = workloads.device_rows(w, n, dev)
    out = torch.empty_like(x)
    peak, _ = hbm_peak()
    res = {"n_vec": n, "D": D}
    for G in (32, 64):
        pk = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty((n, D // G), dtype=torch.float16, device=dev)
        q_ms = _event_ms(torch, stream, lambda: kvq.quantize(
            x, lt, st, G, packed=pk, scales=sc, stream=stream), 10)
        d_ms = _event_ms(torch, stream, lambda: kvq.dequantize(
            pk, sc, lt, st, G, out=out, stream=stream), 10)
        bpv = bytes_per_vector(D, G)
        qg, dg = bpv * n / (q_ms / 1e3) / 1e9, bpv * n / (d_ms / 1e3) / 1e9
        res[f"g{G}"] = {
            "bytes_per_vector": bpv,
            "quantize_ms": round(q_ms, 4), "quantize_gvec_s": round(n / (q_ms / 1e3) / 1e9, 3),
            "quantize_gbs": round(qg, 1), "quantize_frac_of_peak": round(qg / peak, 4),
            "dequantize_ms": round(d_ms, 4), "dequantize_gvec_s": round(n / (d_ms / 1e3) / 1e9, 3),
            "dequantize_gbs": round(dg, 1), "dequantize_frac_of_peak": round(dg / peak, 4),
        }
        del pk, sc
    del x, out
    torch.cuda.empty_cache()
    return res


def run_variants(torch, kvq, dev, stream, x, out, s_t, G, w):
    """The codec's format variants (and the SRFT rotation with lambda after it,
    the paper's configuration) on the same batch, with one lambda table per
    (layer, K/V, head): 36 x 2 x 8 = 576 tables of 128 channels, each over the
    32,768 rows of its tokens.  Algorithmic bytes per vector: 2D (fp16 row) +
    code bytes (D/2 or D) + 2D/G (scales), read once and written once."""
    import numpy as np
    n, D = x.shape
    shape = w.shape or {}
    rows = int(shape.get("tokens", n))
    ntab = max(1, n // rows)
    gen = np.random.default_rng(w.seed + 100)
    tables = torch.from_numpy(gen.uniform(0.5, 2.0, (ntab, D)).astype(np.float32)).to(dev)
    peak, _ = hbm_peak()
    res = {"lambda_tables": ntab, "rows_per_table": rows}
    for bits, after, srft in ((4, True, False), (8, False, False), (8, True, False),
                              (4, True, True)):
        cb = D // 2 if bits == 4 else D
        codes = torch.empty((n, cb), dtype=torch.uint8, device=dev)
        scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
        with ClockSampler(dev.index) as clk:
            q_ms = _event_ms(torch, stream, lambda: kvq.quantize_ex(
                x, tables, s_t, G, bits=bits, lambda_after=after, lambda_rows=rows,
                codes=codes, scales=scales, stream=stream, srft=srft), 10)
            d_ms = _event_ms(torch, stream, lambda: kvq.dequantize_ex(
                codes, scales, tables, s_t, G, bits=bits, lambda_after=after, lambda_rows=rows,
                out=out, stream=stream, srft=srft), 10)
        bpv = 2 * D + cb + 2 * (D // G)
        qg, dg = bpv * n / (q_ms / 1e3) / 1e9, bpv * n / (d_ms / 1e3) / 1e9
        name = f"int{bits}_lambda_{'after' if after else 'before'}" + ("_srft" if srft else "")
        res[name] = {
            "bytes_per_vector": bpv,
            "quantize_ms": round(q_ms, 4), "quantize_gbs": round(qg, 1),
            "quantize_frac_of_peak": round(qg / peak, 4),
            "dequantize_ms": round(d_ms, 4), "dequantize_gbs": round(dg, 1),
            "dequantize_frac_of_peak": round(dg / peak, 4),
            "sm_mhz": clk.summary()["sm_mhz"],
        }
        del codes, scales
    return res


def run_dequant_tc(torch, kvq, dev, stream, x, out, lam_t, s_t):
    """The dequantizer with the in-group Hadamard on the tensor cores beside
    the butterfly dequantizer, on the same batch for G = 16, 32, 64: times,
    HBM fraction, and whether the two outputs are the same bytes."""
    n, D = x.shape
    peak, _ = hbm_peak()
    res = {}
    out2 = torch.empty_like(out)
    for G in (16, 32, 64):
        pk, sc = kvq.quantize(x, lam_t, s_t, G, stream=stream)
        b_ms = _event_ms(torch, stream, lambda: kvq.dequantize(
            pk, sc, lam_t, s_t, G, out=out, stream=stream), 10)
        t_ms = _event_ms(torch, stream, lambda: kvq.dequantize(
            pk, sc, lam_t, s_t, G, out=out2, stream=stream, tensor_cores=True), 10)
        torch.cuda.synchronize()
        bpv = 2 * D + D // 2 + 2 * (D // G)
        bg, tg = bpv * n / (b_ms / 1e3) / 1e9, bpv * n / (t_ms / 1e3) / 1e9
        res[f"G{G}"] = {
            "butterfly_ms": round(b_ms, 4), "butterfly_frac_of_peak": round(bg / peak, 4),
            "tensor_core_ms": round(t_ms, 4), "tensor_core_frac_of_peak": round(tg / peak, 4),
            "same_bytes": bool(torch.equal(out.view(torch.int16), out2.view(torch.int16))),
        }
        del pk, sc
    del out2
    return res


def run_srft_lengths(torch, kvq, dev, stream, G=32, in_bytes=1 << 31):
    """The paper's codec configuration (SRFT rotation, lambda after it, int4
    codes; \"When Quantization Is Free\", technical summary, Methodologie 1-2)
    at every length it runs: D = 64, 96 (mixed radix), 128 and 256, on 2 GiB
    of fp16 rows each (above L2), one lambda table.  Algorithmic bytes per
    vector: 2D + D/2 + 2D/G."""
    import numpy as np
    peak, _ = hbm_peak()
    res = {"group": G, "fp16_input_bytes": in_bytes}
    for D in (64, 96, 128, 256):
        n = in_bytes // (2 * D)
        gen = torch.Generator(device=dev).manual_seed(D)
        x = (torch.randn((n, D), generator=gen, device=dev) * 2.0).to(torch.float16)
        rng = np.random.default_rng(D)
        lam = torch.from_numpy(rng.uniform(0.5, 2.0, D).astype(np.float32)).to(dev)
        sg = torch.from_numpy(np.where(rng.random(D) < 0.5, -1, 1).astype(np.int8)).to(dev)
        codes = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
        out = torch.empty_like(x)
        with ClockSampler(dev.index) as clk:
            q_ms = _event_ms(torch, stream, lambda: kvq.quantize_ex(
                x, lam, sg, G, lambda_after=True, srft=True, codes=codes, scales=scales,
                stream=stream), 10)
            d_ms = _event_ms(torch, stream, lambda: kvq.dequantize_ex(
                codes, scales, lam, sg, G, lambda_after=True, srft=True, out=out, stream=stream), 10)
        bpv = bytes_per_vector(D, G)
        qg, dg = bpv * n / (q_ms / 1e3) / 1e9, bpv * n / (d_ms / 1e3) / 1e9
        res[f"d{D}"] = {
            "n_vec": n, "bytes_per_vector": bpv,
            "quantize_ms": round(q_ms, 4), "quantize_gvec_s": round(n / (q_ms / 1e3) / 1e9, 3),
            "quantize_gbs": round(qg, 1), "quantize_frac_of_peak": round(qg / peak, 4),
            "dequantize_ms": round(d_ms, 4), "dequantize_gvec_s": round(n / (d_ms / 1e3) / 1e9, 3),
            "dequantize_gbs": round(dg, 1), "dequantize_frac_of_peak": round(dg / peak, 4),
            "sm_mhz": clk.summary()["sm_mhz"],
        }
        del x, codes, scales, out
        torch.cuda.empty_cache()
    return res


def run_sustained(torch, kvq, dev, stream, x, out, lam_t, s_t, G, seconds=1.5):
    """Quantize and dequantize of the main batch back to back for about
    `seconds`, each launch timed by CUDA events: the sustained figure under
    the board's power cap, with the SM clocks sampled during the loop."""
    n, D = x.shape
    packed = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
    kvq.quantize(x, lam_t, s_t, G, packed=packed, scales=scales, stream=stream)
    kvq.dequantize(packed, scales, lam_t, s_t, G, out=out, stream=stream)
    torch.cuda.synchronize(dev)
    # size the loop from one timed pair
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    kvq.quantize(x, lam_t, s_t, G, packed=packed, scales=scales, stream=stream)
    kvq.dequantize(packed, scales, lam_t, s_t, G, out=out, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    reps = max(20, int(seconds * 1e3 / max(t0.elapsed_time(t1), 1e-3)))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps + 1)]
    with ClockSampler(dev.index) as clocks:
        ev[0].record(stream)
        for i in range(reps):
            kvq.quantize(x, lam_t, s_t, G, packed=packed, scales=scales, stream=stream)
            ev[2 * i + 1].record(stream)
            kvq.dequantize(packed, scales, lam_t, s_t, G, out=out, stream=stream)
            ev[2 * i + 2].record(stream)
        torch.cuda.synchronize(dev)
    qt = sorted(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(reps))
    dt = sorted(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(reps))
    total_s = ev[0].elapsed_time(ev[-1]) / 1e3
    bpv = bytes_per_vector(D, G)
    qm, dm = qt[len(qt) // 2], dt[len(dt) // 2]
    del packed, scales
    return {
        "reps": reps, "seconds": round(total_s, 3),
        "quantize_ms_median": round(qm, 5), "dequantize_ms_median": round(dm, 5),
        "quantize_gbs": round(bpv * n / (qm / 1e3) / 1e9, 1),
        "dequantize_gbs": round(bpv * n / (dm / 1e3) / 1e9, 1),
        "clocks": clocks.summary(),
    }


DECODE_HQ, DECODE_HKV, DECODE_T = 32, 8, 4096


def build_decode_cache(torch, kvq, dev, stream, lam_t, s_t, G, seqs=64):
    """The int4 cache of the decode configuration: 64 sequences x 36 layers
    (folded into the batch B) x 8 KV heads x 4096 positions, K and V, D = 128,
    holding real quantize output of N(0,1) rows (`seqs` other than 64 only
    for small profiling runs).  Codes [2][B][Hkv][T][D/2] and scales
    [2][B][Hkv][T][D/G], index 0 = K, 1 = V."""
    c = workloads.WORKLOADS["decode-cache"]
    B, Hkv, T, D = seqs * 36, DECODE_HKV, DECODE_T, 128
    rows = 2 * B * Hkv * T
    pk = torch.empty((2, B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((2, B, Hkv, T, D // G), dtype=torch.float16, device=dev)
    pk2, sc2 = pk.view(rows, D // 2), sc.view(rows, D // G)
    chunk = 1 << 23
    buf = torch.empty((chunk, D), dtype=torch.float16, device=dev)
    for i, a in enumerate(range(0, rows, chunk)):
        b = min(rows, a + chunk)
        xr = workloads.device_rows(c, b - a, dev, seed_offset=i, out=buf[: b - a])
        kvq.quantize(xr, lam_t, s_t, G, packed=pk2[a:b], scales=sc2[a:b], stream=stream)
    del buf
    return pk, sc


def run_attention(torch, kvq, dev, stream, lam_t, s_t, G, cache):
    """One decode step of attention over the whole int4 cache of the decode
    configuration (32 query heads on 8 KV heads, Qwen3-8B's grouping).
    Algorithmic bytes: every K and V code and scale once, plus q and the
    output."""
    c = workloads.WORKLOADS["decode-cache"]
    pk, sc = cache
    _, B, Hkv, T, _ = pk.shape
    Hq, D = DECODE_HQ, 128
    kp, vp, ks, vs = pk[0], pk[1], sc[0], sc[1]
    rows = B * Hkv * T
    gen = torch.Generator(device=dev)
    gen.manual_seed(c.seed)
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    need = kvq.kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, G)
    ws = torch.empty(max(need, 0), dtype=torch.uint8, device=dev) if need > 0 else False
    scale = 1.0 / math.sqrt(D)
    ms = _event_ms(torch, stream, lambda: kvq.attention_decode(
        q, kp, ks, vp, vs, lens, lam_t, s_t, lam_t, s_t, G, scale, out=out,
        workspace=ws, stream=stream), 10)
    byts = 2 * rows * (D // 2 + 2 * (D // G)) + 2 * q.numel() * 2
    peak, kind = hbm_peak()
    gbs = byts / (ms / 1e3) / 1e9
    del q, out
    return {
        "shape": f"B={B} ({B // 36} sequences x 36 layers), Hq={Hq}, Hkv={Hkv}, T={T}, D={D}, G={G}",
        "ms": round(ms, 4),
        "algorithmic_bytes": byts,
        "gbs": round(gbs, 1),
        "gkeys_s": round(B * Hkv * T / (ms / 1e3) / 1e9, 2),
        "frac_of_peak": round(gbs / peak, 4),
        "peak_kind": kind,
        "traffic": traffic_per_launch("kvq_attention", rows),
    }


def run_attention_paper_format(torch, kvq, dev, stream, seqs=64):
    """The same decode step over a cache in the paper's own format (SRFT
    rotation, lambda after it, groups of 16: technical summary, Methodologie
    1-3), written by kvq_quantize_ex from the same N(0,1) rows.  Algorithmic
    bytes: every K and V code and scale once (2 x (64 + 16) per row pair),
    plus q and the output."""
    import numpy as np
    c = workloads.WORKLOADS["decode-cache"]
    B, Hkv, T, D, G = seqs * 36, DECODE_HKV, DECODE_T, 128, 16
    Hq = DECODE_HQ
    rows = 2 * B * Hkv * T
    pk = torch.empty((2, B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((2, B, Hkv, T, D // G), dtype=torch.float16, device=dev)
    pk2, sc2 = pk.view(rows, D // 2), sc.view(rows, D // G)
    lam, sgn = workloads.params(D, c.seed + 7)
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(sgn).to(dev)
    chunk = 1 << 23
    buf = torch.empty((chunk, D), dtype=torch.float16, device=dev)
    for i, a in enumerate(range(0, rows, chunk)):
        b = min(rows, a + chunk)
        xr = workloads.device_rows(c, b - a, dev, seed_offset=i, out=buf[: b - a])
        kvq.quantize_ex(xr, lam_t, s_t, G, lambda_after=True, srft=True,
                        codes=pk2[a:b], scales=sc2[a:b], stream=stream)
    del buf
    gen = torch.Generator(device=dev)
    gen.manual_seed(c.seed)
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    scale = 1.0 / math.sqrt(D)
    ms = _event_ms(torch, stream, lambda: kvq.attention_decode(
        q, pk[0], sc[0], pk[1], sc[1], lens, lam_t, s_t, lam_t, s_t, G, scale, out=out,
        stream=stream, lambda_after=True, srft=True), 10)
    byts = rows * (D // 2 + 2 * (D // G)) + 2 * q.numel() * 2
    peak, kind = hbm_peak()
    gbs = byts / (ms / 1e3) / 1e9
    del q, out, pk, sc
    torch.cuda.empty_cache()
    return {
        "shape": f"B={B} ({seqs} sequences x 36 layers), Hq={Hq}, Hkv={Hkv}, T={T}, D={D}, G={G}, "
                 "SRFT, lambda after",
        "ms": round(ms, 4), "algorithmic_bytes": byts, "gbs": round(gbs, 1),
        "frac_of_peak": round(gbs / peak, 4), "peak_kind": kind,
    }


def run_attention_gemma(torch, kvq, dev, stream, seqs=64):
    """Decode attention at Gemma-3-1B's shape: D = 256, 4 query heads on one KV
    head, 26 layers (folded into the batch with `seqs` sequences), 4096
    positions, over real quantize output of the gemma-3-1b rows, in the base
    format at G = 32 and in the paper's format (SRFT, lambda after, G = 16).
    Algorithmic bytes: every K and V code and scale once, plus q and the
    output."""
    w = workloads.WORKLOADS["gemma-3-1b"]
    D, Hq, Hkv, T = 256, 4, 1, 4096
    B = seqs * 26
    rows = 2 * B * Hkv * T
    lam, sgn = workloads.params(D, w.seed + 11)
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(sgn).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    peak, kind = hbm_peak()
    res = {"shape": f"B={B} ({seqs} sequences x 26 layers), Hq={Hq}, Hkv={Hkv}, T={T}, D={D}"}
    chunk = 1 << 22
    buf = torch.empty((chunk, D), dtype=torch.float16, device=dev)
    for name, G, fmt in (("g32", 32, False), ("paper_format_g16", 16, True)):
        pk = torch.empty((2, B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty((2, B, Hkv, T, D // G), dtype=torch.float16, device=dev)
        pk2, sc2 = pk.view(rows, D // 2), sc.view(rows, D // G)
        for i, a in enumerate(range(0, rows, chunk)):
            b = min(rows, a + chunk)
            xr = workloads.device_rows(w, b - a, dev, seed_offset=i, out=buf[: b - a])
            if fmt:
                kvq.quantize_ex(xr, lam_t, s_t, G, lambda_after=True, srft=True,
                                codes=pk2[a:b], scales=sc2[a:b], stream=stream)
            else:
                kvq.quantize(xr, lam_t, s_t, G, packed=pk2[a:b], scales=sc2[a:b], stream=stream)
        ms = _event_ms(torch, stream, lambda: kvq.attention_decode(
            q, pk[0], sc[0], pk[1], sc[1], lens, lam_t, s_t, lam_t, s_t, G, 1.0 / math.sqrt(D),
            out=out, stream=stream, lambda_after=fmt, srft=fmt), 10)
        byts = rows * (D // 2 + 2 * (D // G)) + 2 * q.numel() * 2
        gbs = byts / (ms / 1e3) / 1e9
        res[name] = {"G": G, "ms": round(ms, 4), "algorithmic_bytes": byts, "gbs": round(gbs, 1),
                     "frac_of_peak": round(gbs / peak, 4), "peak_kind": kind}
        del pk, sc
    del buf, q, out
    torch.cuda.empty_cache()
    return res


def run_decode_step(torch, kvq, dev, stream, lam_t, s_t, G, cache, steps=1000):
    """The decode step of the dequantize-then-attend path on the same cache:
    append one new K and V token per (sequence, layer, KV head) into its slot
    (kvq_quantize_rows, 2 x B x 8 = 36,864 vectors at 64 sequences), then
    dequantize the whole cache (150,994,944 vectors) into one reused fp16
    buffer (38.7 GB).  Per-step CUDA-event times, p50 and p99."""
    pk, sc = cache
    two, B, Hkv, T, half = pk.shape
    D = 2 * half
    rows = two * B * Hkv * T
    pk2, sc2 = pk.view(rows, D // 2), sc.view(rows, D // G)
    a = workloads.WORKLOADS["decode-append"]
    na = two * B * Hkv
    xa = workloads.device_rows(a, na, dev)
    base = torch.arange(na, device=dev, dtype=torch.int64) * T
    idx = [base + (p % T) for p in range(8)]
    out = torch.empty((rows, D), dtype=torch.float16, device=dev)

    def one(i):
        kvq.quantize_rows(xa, lam_t, s_t, G, idx[i % 8], pk2, sc2, stream=stream)

    one(0)
    kvq.dequantize(pk2, sc2, lam_t, s_t, G, out=out, stream=stream)
    torch.cuda.synchronize()
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    for i, (e0, e1, e2) in enumerate(ev):
        e0.record(stream)
        one(i)
        e1.record(stream)
        kvq.dequantize(pk2, sc2, lam_t, s_t, G, out=out, stream=stream)
        e2.record(stream)
    torch.cuda.synchronize()
    ap = sorted(e0.elapsed_time(e1) for e0, e1, _ in ev)
    dq = sorted(e1.elapsed_time(e2) for _, e1, e2 in ev)
    pct = lambda t, p: t[min(len(t) - 1, int(p * len(t)))]
    bpv = bytes_per_vector(D, G)
    peak, _ = hbm_peak()
    del xa, out
    torch.cuda.empty_cache()
    return {
        "steps": steps, "append_vectors": na, "cache_vectors": rows,
        "append_us_p50": round(pct(ap, 0.5) * 1e3, 2), "append_us_p99": round(pct(ap, 0.99) * 1e3, 2),
        "dequant_ms_p50": round(pct(dq, 0.5), 4), "dequant_ms_p99": round(pct(dq, 0.99), 4),
        "dequant_gvec_s": round(rows / (pct(dq, 0.5) / 1e3) / 1e9, 3),
        "dequant_gbs": round(bpv * rows / (pct(dq, 0.5) / 1e3) / 1e9, 1),
        "dequant_frac_of_peak": round(bpv * rows / (pct(dq, 0.5) / 1e3) / 1e9 / peak, 4),
    }


def run_e2e(args, torch, kvq, dev, x_dev, lam_t, s_t, G, world):
    """Host fp16 batch -> device -> quantize -> dequantize -> host fp16, per step,
    chunked over three streams so that H2D, compute and D2H of different chunks
    overlap.  Device-timed (events on the copy streams) and max over ranks."""
    n, D = x_dev.shape
    chunks = args.e2e_chunks
    bounds = [(n * i) // chunks for i in range(chunks + 1)]
    host_in = torch.empty((n, D), dtype=torch.float16, pin_memory=True)
    host_in.copy_(x_dev, non_blocking=False)
    host_out = torch.empty((n, D), dtype=torch.float16, pin_memory=True)
    d_in = torch.empty_like(x_dev)
    d_out = torch.empty_like(x_dev)
    d_packed = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    d_scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
    s_h2d, s_comp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))

    def one_step():
        for i in range(chunks):
            a, b = bounds[i], bounds[i + 1]
            e_in = torch.cuda.Event()
            with torch.cuda.stream(s_h2d):
                d_in[a:b].copy_(host_in[a:b], non_blocking=True)
                e_in.record(s_h2d)
            s_comp.wait_event(e_in)
            kvq.quantize(d_in[a:b], lam_t, s_t, G, packed=d_packed[a:b],
                         scales=d_scales[a:b], stream=s_comp)
            kvq.dequantize(d_packed[a:b], d_scales[a:b], lam_t, s_t, G,
                           out=d_out[a:b], stream=s_comp)
            e_c = torch.cuda.Event()
            e_c.record(s_comp)
            s_d2h.wait_event(e_c)
            with torch.cuda.stream(s_d2h):
                host_out[a:b].copy_(d_out[a:b], non_blocking=True)

    one_step()
    torch.cuda.synchronize(dev)
    K = max(1, min(args.steps, args.e2e_steps))
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    start.record(s_h2d)
    s_comp.wait_event(start)
    s_d2h.wait_event(start)
    for _ in range(K):
        one_step()
    s_d2h.wait_stream(s_h2d)
    s_d2h.wait_stream(s_comp)
    end.record(s_d2h)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    ok = bool(torch.equal(host_out[:4096].to(dev), d_out[:4096]))
    return {"value": round(n * world * K / (ms / 1e3) / 1e9, 4), "unit": UNIT,
            "h2d_bytes_per_step": n * D * 2, "d2h_bytes_per_step": n * D * 2,
            "steps": K, "ms_per_step": round(ms / K, 3), "chunks": chunks,
            "result_copied_back": ok}


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle, as it stands, on the host's cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    w = workloads.WORKLOADS[args.workload]
    G = args.group or w.groups[0]
    ot = OracleTimer(w, G, args.ref_step_seconds)
    times = [ot.run() for _ in range(args.warmup + args.steps)][args.warmup:]
    tot_s = sum(times)
    value = ot.rows * len(times) / tot_s / 1e9
    rows, threads = ot.rows, ot.threads
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_s / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "n_vec_per_gpu": w.n_vec, "D": w.D, "group": G,
                   "shape": w.shape, "values": w.note,
                   "sample_per_step": f"{rows} vectors (bounded sample of the workload)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} vectors per step, quantize+dequantize"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def parse(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="qwen3-8b-prefill", choices=sorted(workloads.WORKLOADS))
    p.add_argument("--group", type=int, default=None)
    p.add_argument("--n-vec", type=int, default=None, help="override vectors per GPU (profiling)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip round-trip, append and attention figures")
    p.add_argument("--attention-only", action="store_true",
                   help="of the secondary figures, only the decode attention (profiling)")
    p.add_argument("--variants-only", action="store_true",
                   help="of the secondary figures, only the codec variants (profiling)")
    p.add_argument("--configs-only", action="store_true",
                   help="of the secondary figures, only the smaller configurations (profiling)")
    p.add_argument("--tc-only", action="store_true",
                   help="of the secondary figures, only the tensor-core dequantizer (profiling)")
    p.add_argument("--roundtrip-only", action="store_true",
                   help="of the secondary figures, only the fused round trip (profiling)")
    p.add_argument("--attn-seqs", type=int, default=64, help="sequences of the attention figure (profiling)")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--e2e-chunks", type=int, default=16)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-step-seconds", type=float, default=2.0)
    args = p.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours" and args.n_vec is None:
        p.error("--warmup must be >= 3")
    return args


def main(argv=None):
    args = parse(argv)
    line = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
