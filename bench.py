#!/usr/bin/env python
"""Decode-attention throughput of the packed Block-GTQ cache on B200.

One step = one decode step of the whole model: for every layer, append the
step's new token to the packed cache (TQ-MSE encode of its K and V rows at
position len-1, so lengths stay fixed) and run GQA decode attention over the
packed cache (query rotation, split-K pass, split merge and inverse V
rotation: one fused launch).  Steps run as one CUDA graph.
value = sequences * steps / time (decode tokens/s).

Printed as one JSON line on rank 0.  Also measured in the same run:
  roofline      the fused decode kernel: its per-layer launches back to back
                in a captured graph (launch_ms) and with events around each
                launch inside a captured step (launch_ms_isolated), against
                the measured HBM peak
  e2e           the same step through the C ABI from pinned host buffers (H2D
                of the queries and new K/V, D2H of the outputs inside the timing)
  multi_layer   all layers in one launch per kernel
  buffered      the step with 4 fp16 sink rows and a 128-row fp16 window
  paged         the step on a paged copy of the cache (shuffled pages)
  logit_mae     per-layer logit MAE, Block-GTQ against uniform TQ-MSE
  fp16_baseline dense fp16 decode over the unquantised K/V: FlashAttention-2's
                decode with its split count swept, and torch SDPA; the best
                one with its HBM fraction
  cpu_baseline  the CPU oracle on a bounded sample (rank 0, one GPU),
                extrapolated to a step and labelled so
  workloads     (one GPU) the other benchmark shapes -- tiny, llama, batch,
                long -- each with its step, roofline, fp16 baseline, CPU
                baseline and compression; long adds the 131072-row prefill
                chunk's encode rate

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen3b]
  python bench.py --impl reference ...   (the CPU oracle as the reference arm)
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
SIDE_WORKLOADS = ("tiny", "llama", "batch", "long")

# DRAM bytes (read + write) per launch of the decode kernel from an ncu
# capture, per workload, with the date of the capture and a digest of the
# kernel sources it was taken on.  The roofline reports it only while the
# sources still match that digest (null otherwise: the kernel has changed).
NCU_TRAFFIC = {
    "qwen3b": {"bytes_per_launch": 27897344, "captured": "2026-12-02",
               "case": "8 of the 36 layers, the same per-layer split launch; dram__bytes_read.sum 27.90 MB, "
                       "dram__bytes_write.sum 0; decode.cu's header comments edited since (sources digest "
                       "2944aa7cf6d47af1 at the capture), no code change",
               "kernel_digest": "69fdba149f4e04c1"},
}
KERNEL_SOURCES = ("packed_decode_attention_b200/csrc/decode.cu", "packed_decode_attention_b200/csrc/common.cuh",
                  "packed_decode_attention_b200/csrc/device_tables.h")


def kernel_digest():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3b")
    ap.add_argument("--layers", type=int, default=0, help="use only the first N layers (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp16-baseline", action="store_true")
    ap.add_argument("--no-diag", action="store_true", help="skip the per-layer logit-MAE diagnostic")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged-cache step")
    ap.add_argument("--no-side", action="store_true", help="skip the other workloads (the workloads object)")
    ap.add_argument("--decode-path", type=int, default=-1, choices=[-1, 0, 1],
                    help="1: fused decode launch, 0: rotation + split + combine, -1: the library's default")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def barrier(world):
    """All ranks meet (no-op for one process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    """The largest x over all ranks (a step time: the job is as slow as its
    slowest replica).  device: where the process group's tensors live (a
    CUDA device under NCCL, the CPU under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, batch, ms_step):
    """Whole-job throughput: every rank decodes its own batch (weak scaling)."""
    return world * batch / (ms_step * 1e-3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def cpu_cores():
    """Host cores this process may run on (its CPU affinity)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return max(1, os.cpu_count() or 1)


class ClockSampler:
    """SM clock and clock-event reasons sampled while running: NVML polled
    every millisecond from a thread (read-only queries), else nvidia-smi
    at its 200 ms minimum."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid, device_index):
        self.uuid = device_uuid
        self.index = device_index
        self.samples = []          # (time, sm_mhz, max_mhz, reasons set)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            masks = [(n, getattr(pynvml, m)) for n, m in self.REASONS]
            max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)

            def poll():
                while not self.stop_flag.is_set():
                    mhz = pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    self.samples.append((time.time(), float(mhz), float(max_mhz), {n for n, m in masks if r & m}))
                    time.sleep(0.001)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 7:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]),
                                     {n for n, v in zip(names, parts[3:7]) if v.lower() == "active"}))
            except ValueError:
                continue

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [x for x in self.samples if t0 <= x[0] <= t1] or \
            [x for x in self.samples if t0 - 0.25 <= x[0] <= t1 + 0.25]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for x in rows:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in rows), "sm_max_mhz": max(x[2] for x in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


def token_bytes(kv, cfg):
    """Algorithmic packed bytes per cached token for each (layer, KV head)."""
    from packed_decode_attention_b200 import bgtq
    out = {}
    for l in range(cfg.n_layers):
        for h in range(cfg.n_kv_heads):
            ng = bgtq.bgtq_get_layout(kv.state, l, h)[0]
            out[l, h] = 16 * cfg.k_avg_bits + 16 * cfg.v_avg_bits + 2 * ng + 2
    return out


class OracleSample:
    """A bounded sample of the workload for the CPU oracle: a few (layer, KV
    head) pairs of sequence 0 over its first `t_len` cached tokens (at most
    max_tokens), each with its own oracle allocation, tables and packed cache
    (built once, untimed).  One timed unit is the oracle's decode of the G
    query heads of a pair over that cache plus the encode of one new K/V row.
    A full step is every (layer, KV head) of every sequence over all its
    tokens, so the step time is extrapolated from the unit time by the factor
    layers * KV heads * (total cached tokens / t_len); the decode's cost is
    linear in the tokens."""

    def __init__(self, w, lens, max_pairs=4, max_tokens=None):
        import numpy as np

        from oracle import model
        from packed_decode_attention_b200 import workloads as wl

        self.w, self.lens = w, lens
        pairs = [(l, h) for l in range(w.n_layers) for h in range(w.n_kv_heads)]
        self.n_pairs = len(pairs)
        pick = [pairs[i] for i in np.linspace(0, len(pairs) - 1, num=min(max_pairs, len(pairs))).astype(int)]
        self.t_len = lens[0] if max_tokens is None else min(lens[0], max_tokens)
        cfg = model.Config(w.n_layers, w.n_kv_heads, w.n_q_heads, 128, w.k_bits, w.v_bits, 1, 4, 0, w.seed)
        self.units = []
        for (l, h) in pick:
            cq = wl.queries(w, l, 0, np.arange(w.n_calib), tag=1)[None]
            ck = wl.keys(w, l, 0, 0, w.n_calib)[None]
            c1 = model.Config(1, w.n_kv_heads, w.n_q_heads, 128, w.k_bits, w.v_bits, 1, 4, 0, w.seed)
            full = np.zeros((w.n_layers, w.n_kv_heads, 64), dtype=np.int64)
            full[l] = model.allocate(c1, cq.numpy(), ck.numpy())[0]
            tb = model.Tables(cfg, full, layers=[l])
            k = wl.keys(w, l, 0, 0, self.t_len)[:, h].numpy()
            v = wl.values(w, l, 0, 0, self.t_len)[:, h].numpy()
            enc = model.encode_rows(tb, l, h, k, v)
            q = wl.queries(w, l, 0, [self.t_len], tag=2)[0, h * w.group:(h + 1) * w.group].numpy()
            self.units.append((tb, l, h, k[-1:], v[-1:], q, enc))

    @property
    def scale(self):
        """Full step time / one unit's time."""
        w = self.w
        return w.n_layers * w.n_kv_heads * (sum(self.lens) / float(self.t_len))

    def time_unit(self, i):
        from oracle import model
        tb, l, h, k1, v1, q, enc = self.units[i % len(self.units)]
        t0 = time.perf_counter()
        model.encode_rows(tb, l, h, k1, v1)
        model.decode(tb, l, h, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], enc["n"])
        return time.perf_counter() - t0

    def describe(self):
        w = self.w
        return (f"oracle decode of the {w.group} query heads of one (layer, KV head) over {self.t_len} cached "
                f"tokens of sequence 0 + encode of one K/V row, on {len(self.units)} of {self.n_pairs} "
                f"(layer, KV head) pairs; a full step (every pair of all {w.batch} sequences, "
                f"{sum(self.lens)} cached tokens each) is extrapolated as the mean unit time x {self.scale:.6g}")


def oracle_baseline(w, lens, n_units, max_pairs=3, max_tokens=None):
    """The oracle on the host cores (BLAS threads = the process's cores):
    n_units timed units, extrapolated to one step.  Returns (cpu_baseline
    dict, unit seconds list)."""
    import contextlib
    cores = cpu_cores()
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=cores)
    except Exception:
        limiter = contextlib.nullcontext()
    with limiter:
        sample = OracleSample(w, lens, max_pairs=max_pairs, max_tokens=max_tokens)
        units = [sample.time_unit(i) for i in range(n_units)]
    unit_s = statistics.mean(units)
    step_s = unit_s * sample.scale
    return {"value": w.batch / step_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": sample.describe(), "extrapolated": True, "units_timed": len(units),
            "unit_ms": unit_s * 1e3, "scale_to_step": sample.scale, "step_ms_extrapolated": step_s * 1e3}, units


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    from packed_decode_attention_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    lens = wl.seq_lens(w)
    # warm-up units run untimed; each timed step is one unit of the sample
    cores = cpu_cores()
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=cores)
    except Exception:
        pass
    sample = OracleSample(w, lens, max_pairs=2)
    for i in range(args.warmup):
        sample.time_unit(i)
    units = [sample.time_unit(args.warmup + i) for i in range(args.steps)]
    unit_s = statistics.mean(units)
    step_s = unit_s * sample.scale
    value = w.batch / step_s
    line = {
        "impl": "reference", "metric": "decode_tokens_per_s", "value": value, "unit": "tokens/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup, "ms_per_step": unit_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, lens),
        "step_definition": "each step is one unit of the bounded sample (see cpu_baseline.sample); value is "
                           "tokens/s of a full decode step extrapolated from the mean unit time",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample.describe(), "extrapolated": True, "units_timed": len(units),
                         "unit_ms": unit_s * 1e3, "scale_to_step": sample.scale,
                         "step_ms_extrapolated": step_s * 1e3},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, lens):
    return {"workload": f"{w.name}: {w.n_layers} layers x {w.n_kv_heads} KV heads, {w.n_q_heads} q heads, "
                        f"head_dim 128, batch {w.batch} x {max(lens)} cached tokens, K{w.k_bits}V{w.v_bits}",
            "layers": w.n_layers, "kv_heads": w.n_kv_heads, "q_heads": w.n_q_heads, "batch": w.batch,
            "context": max(lens), "total_cached_tokens": int(sum(lens)), "k_bits": w.k_bits, "v_bits": w.v_bits,
            "l2": "inputs larger than L2: every step streams the whole packed cache of all layers",
            "parallelism": "replicas"}


def host_overhead_hidden():
    """Keeps the GPU busy (a ~1 ms spin) while the host issues the call timed
    next, so that events around one eager call measure its kernels and not the
    host-side argument checks in front of them."""
    import torch
    torch.cuda._sleep(2_000_000)


def time_graph(fn, steps, warmup, world=1):
    """Average ms of one call of fn, captured as a CUDA graph and replayed
    `steps` times after `warmup` replays, CUDA events around the timed region.
    Returns (ms, graph, (wall t0, wall t1))."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    a.record()
    for _ in range(steps):
        g.replay()
    z.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    return a.elapsed_time(z) / steps, g, (t_wall0, t_wall1)


def fp16_baseline(w, lens, q_all, kf, vf, seq, steps, warmup, world, dev, peak, ms_packed):
    """Dense fp16 decode over the unquantised K/V: FlashAttention-2's decode
    (flash_attn_with_kvcache) with its split count swept, and torch SDPA
    (flash and cuDNN backends, per sequence); the best one is the baseline."""
    import torch
    import torch.nn.functional as F
    L, B, HQ = w.n_layers, w.batch, w.n_q_heads
    H = w.n_kv_heads
    qf = q_all.view(L, B, 1, HQ, 128)
    step_bytes = int(sum(lens) * H * L * 512 + L * B * HQ * 512)
    cands = []
    try:
        from flash_attn import flash_attn_with_kvcache
        for ns in (0, 2, 4, 8, 16, 32, 64, 128):
            def fa2(ns=ns):
                for l in range(L):
                    flash_attn_with_kvcache(qf[l], kf[l], vf[l], cache_seqlens=seq, num_splits=ns)
            cands.append((f"flash_attn_with_kvcache (FlashAttention-2 decode), num_splits={ns}", fa2))
    except Exception:
        pass
    results = []
    for name, fn in cands:
        try:
            ms, g, _ = time_graph(fn, max(3, steps // 2), max(2, warmup // 2), world)
            del g
            ms = max_over_ranks(ms, world, dev)
            results.append({"impl": name, "ms_per_step": ms})
        except Exception as e:  # report, do not fail the bench
            results.append({"impl": name, "error": str(e)[:160]})
            torch.cuda.synchronize()
    # torch SDPA per sequence, timed eagerly (launched one call at a time)
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for backend, bname in ((SDPBackend.FLASH_ATTENTION, "flash"), (SDPBackend.CUDNN_ATTENTION, "cudnn")):
        def sdpa(backend=backend):
            with sdpa_kernel(backend):
                for l in range(L):
                    for b in range(B):
                        qq = q_all[l, b][None, :, None, :]
                        kk = kf[l][b, :lens[b]].transpose(0, 1)[None]
                        vv = vf[l][b, :lens[b]].transpose(0, 1)[None]
                        F.scaled_dot_product_attention(qq, kk, vv, enable_gqa=True)
        name = f"torch scaled_dot_product_attention ({bname} backend, eager)"
        try:
            for _ in range(2):
                sdpa()
            torch.cuda.synchronize()
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = max(3, steps // 2)
            a.record()
            for _ in range(n):
                sdpa()
            z.record()
            torch.cuda.synchronize()
            results.append({"impl": name, "ms_per_step": max_over_ranks(a.elapsed_time(z) / n, world, dev)})
        except Exception as e:
            results.append({"impl": name, "error": str(e)[:160]})
            torch.cuda.synchronize()
    ok = [r for r in results if "ms_per_step" in r]
    if not ok:
        return {"error": "no fp16 decode ran", "candidates": results}
    best = min(ok, key=lambda r: r["ms_per_step"])
    gbs = step_bytes / (best["ms_per_step"] * 1e-3) / 1e9
    fa2 = [r for r in ok if r["impl"].startswith("flash_attn_with_kvcache")]
    fa2_default = next((r for r in fa2 if r["impl"].endswith("num_splits=0")), None)
    return {"impl": best["impl"], "ms_per_step": best["ms_per_step"],
            "tokens_per_s": world * B / (best["ms_per_step"] * 1e-3), "bytes_per_step": step_bytes,
            "hbm_gbs": gbs, "hbm_frac": gbs / peak, "speedup_of_packed": best["ms_per_step"] / ms_packed,
            "fa2_default_ms": fa2_default["ms_per_step"] if fa2_default else None,
            "candidates": [{k: (round(v, 5) if isinstance(v, float) else v) for k, v in r.items()} for r in results]}


def measure(w, args, dev, world, rank, full):
    """Every figure of one workload.  full: the headline workload (all extras);
    otherwise the step, roofline, fp16 and CPU baselines, compression and
    (long context) the prefill chunk's encode rate."""
    import numpy as np
    import torch

    from packed_decode_attention_b200 import bgtq
    from packed_decode_attention_b200 import workloads as wl

    lens = wl.seq_lens(w)
    L, H, HQ, B = w.n_layers, w.n_kv_heads, w.n_q_heads, w.batch
    cap = w.seq_len
    cfg = bgtq.Config(**wl.bench_config_fields(w))
    kv = bgtq.PackedKVCache(cfg, dev)
    if args.decode_path >= 0:
        kv.set_decode_path(args.decode_path)
    fused = kv.decode_path_fused()
    steps = args.steps if full else max(5, args.steps // 2)
    warmup = args.warmup if full else max(3, args.warmup // 2)
    peak, peak_kind = peaks()

    # ---- calibration + allocation (one-time) ----
    cq, ck = wl.calibration(w, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    kv.allocate(cq, ck)
    e1.record()
    torch.cuda.synchronize()
    alloc_ms = e0.elapsed_time(e1)
    del cq, ck

    # ---- prefill: encode the whole cache (and keep fp16 K/V for the dense baseline) ----
    want_fp16 = not args.no_fp16_baseline
    kf = [torch.empty((B, cap, H, 128), dtype=torch.float16, device=dev) for _ in range(L)] if want_fp16 else None
    vf = [torch.empty((B, cap, H, 128), dtype=torch.float16, device=dev) for _ in range(L)] if want_fp16 else None
    chunk = w.encode_chunk or 32768  # rows per encode call: the long workload's 131072-row prefill chunk
    for l in range(L):
        for b in range(B):
            for s0 in range(0, lens[b], chunk):
                n = min(chunk, lens[b] - s0)
                kk = torch.zeros((1, B, n, H, 128), dtype=torch.float16, device=dev)
                vv = torch.zeros_like(kk)
                kk[0, b] = wl.keys(w, l, b, s0, n, device=dev)
                vv[0, b] = wl.values(w, l, b, s0, n, device=dev)
                if want_fp16:
                    kf[l][b, s0:s0 + n] = kk[0, b]
                    vf[l][b, s0:s0 + n] = vv[0, b]
                start = torch.zeros(B, dtype=torch.int32, device=dev)
                count = torch.zeros(B, dtype=torch.int32, device=dev)
                start[b] = s0
                count[b] = n
                kv.encode_append(l, kk, vv, start, count)
                del kk, vv
    torch.cuda.synchronize()
    assert kv.device_error() == 0, "device error after prefill"
    # prefill rate: one prefill call (the first chunk of layer 0, sequence 0)
    # encoded again -- the same rows, so the same bytes -- as a captured
    # graph replayed back to back (the kernels only, without the host's
    # argument checks)
    n_p = min(chunk, lens[0])
    kk = torch.zeros((1, B, n_p, H, 128), dtype=torch.float16, device=dev)
    vv = torch.zeros_like(kk)
    kk[0, 0] = wl.keys(w, 0, 0, 0, n_p, device=dev)
    vv[0, 0] = wl.values(w, 0, 0, 0, n_p, device=dev)
    st_p = torch.zeros(B, dtype=torch.int32, device=dev)
    cnt_p = torch.zeros(B, dtype=torch.int32, device=dev)
    cnt_p[0] = n_p
    enc_call_ms, g_e, _ = time_graph(lambda: kv.encode_append(0, kk, vv, st_p, cnt_p), 5, 3)
    del g_e, kk, vv
    assert kv.device_error() == 0, "device error in the prefill re-encode"

    # ---- step inputs ----
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    start1 = seq - 1
    count1 = torch.ones(B, dtype=torch.int32, device=dev)
    q_all = torch.stack([wl.decode_query(w, l, lens, device=dev) for l in range(L)])          # [L, B, HQ, 128]
    knew = torch.zeros((L, B, 1, H, 128), dtype=torch.float16, device=dev)
    vnew = torch.zeros_like(knew)
    for l in range(L):
        for b in range(B):
            knew[l, b, 0] = wl.keys(w, l, b, lens[b] - 1, 1, device=dev)[0]
            vnew[l, b, 0] = wl.values(w, l, b, lens[b] - 1, 1, device=dev)[0]
    out = torch.empty((L, B, HQ, 128), dtype=torch.float16, device=dev)

    def step():
        # per layer: append the new K/V row, then attend
        for l in range(L):
            kv.decode_step(l, knew[l:l + 1], vnew[l:l + 1], start1, count1, q_all[l:l + 1], seq, out[l:l + 1])

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid, dev.index or 0)
    sampler.start()
    time.sleep(0.3)
    ms_step, graph, (tw0, tw1) = time_graph(step, steps, warmup, world)
    sampler.stop()
    clocks = sampler.summary(tw0, tw1)
    ms_step = max_over_ranks(ms_step, world, dev)
    assert kv.device_error() == 0, "device error during the timed steps"
    assert torch.isfinite(out.float()).all(), "non-finite decode output"

    # ---- roofline: the decode kernel's average launch duration, its
    # per-layer launches (same inputs, same launch configuration as in the
    # step) back to back in one captured graph ----
    tb = token_bytes(kv, cfg)
    bytes_per_layer = [sum(lens[b] * tb[l, h] for b in range(B) for h in range(H)) + B * HQ * 512 for l in range(L)]
    alg_bytes = statistics.mean(bytes_per_layer)

    def decodes_back_to_back():
        for l in range(L):
            kv.decode_attn(l, q_all[l:l + 1], seq, out[l:l + 1])

    ms_dec, g_d, _ = time_graph(decodes_back_to_back, steps, warmup, world)
    del g_d
    launch_ms = max_over_ranks(ms_dec / L, world, dev)
    achieved = alg_bytes / (launch_ms * 1e-3) / 1e9

    # the same launches with events around each one inside a captured step
    # (the event nodes keep it from overlapping its neighbours: start-up included)
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(L)]

    def step_timed():
        for l in range(L):
            kv.encode_append(l, knew[l:l + 1], vnew[l:l + 1], start1, count1)
            ev[l][0].record()
            kv.decode_attn(l, q_all[l:l + 1], seq, out[l:l + 1])
            ev[l][1].record()

    step_timed()
    torch.cuda.synchronize()
    g_t = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_t):
        step_timed()
    iso = []
    for it in range(warmup + steps):
        g_t.replay()
        torch.cuda.synchronize()
        if it >= warmup:
            iso.extend(a.elapsed_time(z) for a, z in ev)
    del g_t
    launch_ms_isolated = statistics.mean(iso)

    digest = kernel_digest()
    cap_rec = NCU_TRAFFIC.get(w.name)
    traffic = cap_rec["bytes_per_launch"] if cap_rec and cap_rec.get("kernel_digest") == digest else None
    traffic_source = (f"ncu capture of {cap_rec['captured']} ({cap_rec['case']}), same kernel sources"
                      if traffic is not None else "no ncu capture of the current kernel sources")
    decode_call = {"launch_ms": launch_ms, "launch_ms_isolated": launch_ms_isolated, "achieved_gbs": achieved,
                   "frac": achieved / peak,
                   "kernels": "decode_fused_kernel" if fused else "rotate_query_kernel + decode_mma_kernel + combine_kernel",
                   "timing": "launch_ms: the step's per-layer bgtq_decode_attn calls back to back in a captured "
                             "graph, events around the region / calls; launch_ms_isolated: events around each call "
                             "inside a captured step (start-up not overlapped)"}
    if fused:
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": traffic, "traffic_source": traffic_source, "kernel": "decode_fused_kernel",
                    "launch_ms": launch_ms, "alg_bytes_per_launch": alg_bytes, "peak_kind": peak_kind,
                    "kernel_digest": digest, "timing": decode_call["timing"]}
    else:
        # the dominant kernel alone: the split pass's per-layer launches
        # (bgtq_decode_split on the step's rotated queries) back to back
        qrot_all = torch.empty((L, B, HQ, 128), dtype=torch.float32, device=dev)
        for l in range(L):
            kv.rotate_query(l, q_all[l:l + 1], qrot_all[l:l + 1])

        def splits_back_to_back():
            for l in range(L):
                kv.decode_split(l, qrot_all[l:l + 1], seq)

        ms_sp, g_sp, _ = time_graph(splits_back_to_back, steps, warmup, world)
        del g_sp, qrot_all
        sp_ms = max_over_ranks(ms_sp / L, world, dev)
        sp_bytes = alg_bytes - B * HQ * 512  # the packed cache only (q and o are the other kernels')
        sp_gbs = sp_bytes / (sp_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": sp_gbs, "peak": peak, "unit": "GB/s", "frac": sp_gbs / peak,
                    "traffic": traffic, "traffic_source": traffic_source, "kernel": "decode_mma_kernel",
                    "launch_ms": sp_ms, "alg_bytes_per_launch": sp_bytes, "peak_kind": peak_kind,
                    "kernel_digest": digest,
                    "timing": "launch_ms: the split pass's per-layer launches (bgtq_decode_split) back to back "
                              "in a captured graph, events around the region / launches"}
    step_bytes = sum(bytes_per_layer)
    res = {"ms_per_step": ms_step, "tokens_per_s": world * B / (ms_step * 1e-3),
           "step_hbm_gbs": step_bytes / (ms_step * 1e-3) / 1e9, "roofline": roofline, "decode_call": decode_call,
           "clocks": clocks,
           "decode_path": "fused (one launch per decode call)" if fused else "query rotation + split + combine",
           "decode_wave_ctas": kv.decode_wave_ctas(),
           "gpu_launches": (2 if fused else 3) * L * steps,
           "allocate_ms": alloc_ms, "prefill_encode_rows_per_s": n_p * H / (enc_call_ms * 1e-3),
           "prefill_encode_call_rows": n_p, "prefill_encode_call_ms": enc_call_ms,
           "compression_vs_fp16": 512.0 / (sum(lens[b] * tb[l, h] for l in range(L) for b in range(B)
                                                for h in range(H)) / (sum(lens) * L * H))}

    if full:
        # ---- end to end from pinned host memory ----
        q_h = q_all.cpu().pin_memory()
        k_h = knew.cpu().pin_memory()
        v_h = vnew.cpu().pin_memory()
        o_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = q_h.numel() * 2 + k_h.numel() * 2 + v_h.numel() * 2
        d2h = o_h.numel() * 2
        for _ in range(warmup):
            q_all.copy_(q_h, non_blocking=True)
            knew.copy_(k_h, non_blocking=True)
            vnew.copy_(v_h, non_blocking=True)
            graph.replay()
            o_h.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            q_all.copy_(q_h, non_blocking=True)
            knew.copy_(k_h, non_blocking=True)
            vnew.copy_(v_h, non_blocking=True)
            graph.replay()
            o_h.copy_(out, non_blocking=True)
        z.record()
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(a.elapsed_time(z) / steps, world, dev)
        res["e2e"] = {"value": world * B / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h}

        # ---- all layers in one launch per kernel ----
        def step_multi():
            kv.encode_append(0, knew, vnew, start1, count1, layer_count=L)
            kv.decode_attn(0, q_all, seq, out, layer_count=L)

        ms_multi, g_m, _ = time_graph(step_multi, steps, warmup, world)
        del g_m
        ms_multi = max_over_ranks(ms_multi, world, dev)
        ml_gbs = step_bytes / (ms_multi * 1e-3) / 1e9
        res["multi_layer"] = {"ms_per_step": ms_multi, "tokens_per_s": world * B / (ms_multi * 1e-3),
                              "hbm_gbs": ml_gbs, "frac": ml_gbs / peak,
                              "note": "the same step with all layers in one launch per kernel (appends, then "
                                      "rotation + split + combine): the kernels without per-layer launch "
                                      "granularity; a model cannot batch its layers like this"}

        # ---- fp16 sink + recent window (the README's "withbuffer" setting) ----
        SINK, WINDOW = 4, 128
        lo_b = [min(SINK, n) for n in lens]
        hi_b = [max(lo_b[b], lens[b] - WINDOW) for b in range(B)]
        n_buf = SINK + WINDOW
        buf_k = torch.zeros((L, B, n_buf, H, 128), dtype=torch.float16, device=dev)
        buf_v = torch.zeros_like(buf_k)
        for l in range(L):
            for b in range(B):
                rows = list(range(lo_b[b])) + list(range(hi_b[b], lens[b]))
                for j, r in enumerate(rows):
                    buf_k[l, b, j] = wl.keys(w, l, b, r, 1, device=dev)[0]
                    buf_v[l, b, j] = wl.values(w, l, b, r, 1, device=dev)[0]
        buf_cnt = torch.tensor([lo_b[b] + lens[b] - hi_b[b] for b in range(B)], dtype=torch.int32, device=dev)
        seq_hi = torch.tensor(hi_b, dtype=torch.int32, device=dev)
        seq_lo = torch.tensor(lo_b, dtype=torch.int32, device=dev)

        def step_buffered():
            for l in range(L):
                kv.decode_step_buffered(l, knew[l:l + 1], vnew[l:l + 1], start1, count1, q_all[l:l + 1], seq_hi,
                                        seq_lo, buf_k[l:l + 1], buf_v[l:l + 1], buf_cnt, out[l:l + 1])

        ms_buf, g_buf, _ = time_graph(step_buffered, steps, warmup, world)
        ms_buf = max_over_ranks(ms_buf, world, dev)
        del g_buf, buf_k, buf_v
        assert kv.device_error() == 0, "device error in the buffered step"
        res["buffered"] = {"ms_per_step": ms_buf, "tokens_per_s": world * B / (ms_buf * 1e-3), "sink": SINK,
                           "window": WINDOW, "note": "fp16 sink + recent window next to the packed cache "
                                                     "(query rotation, split pass with buffer CTAs, combine)"}

        # ---- the same step over a paged copy of the cache ----
        if not args.no_paged:
            T = (cap + 63) // 64
            need = [(n + 63) // 64 for n in lens]
            pool = sum(need)
            ids = torch.randperm(pool, generator=torch.Generator().manual_seed(7)).to(torch.int32)
            table = torch.full((B, T), -1, dtype=torch.int32)
            k0 = 0
            for b in range(B):
                table[b, :need[b]] = ids[k0:k0 + need[b]]
                k0 += need[b]
            bt = table.to(dev)
            kvp = bgtq.PackedKVCache(bgtq.Config(**dict(wl.bench_config_fields(w), page_pool_tiles=pool)), dev)
            kvp.set_block_table(bt)
            kvp.set_allocation(kv.get_allocation())
            for l in range(L):
                for b in range(B):
                    pg = bt[b, :need[b]].long()
                    for h in range(H):
                        kvp.k_tiles()[l, h][pg] = kv.k_tiles()[l, b, h, :need[b]]
                        kvp.v_tiles()[l, h][pg] = kv.v_tiles()[l, b, h, :need[b]]
                        kvp.k_norms()[l, h].view(pool, 64, 4)[pg] = kv.k_norms()[l, b, h, :need[b] * 64].view(-1, 64, 4)
                        kvp.v_norms()[l, h].view(pool, 64)[pg] = kv.v_norms()[l, b, h, :need[b] * 64].view(-1, 64)
            out_p = torch.empty_like(out)

            def step_paged():
                for l in range(L):
                    kvp.decode_step(l, knew[l:l + 1], vnew[l:l + 1], start1, count1, q_all[l:l + 1], seq,
                                    out_p[l:l + 1])

            ms_paged, g_p, _ = time_graph(step_paged, steps, warmup, world)
            ms_paged = max_over_ranks(ms_paged, world, dev)
            del g_p
            step()
            step_paged()
            torch.cuda.synchronize()
            assert kvp.device_error() == 0, "device error in the paged step"
            res["paged"] = {"ms_per_step": ms_paged, "tokens_per_s": world * B / (ms_paged * 1e-3), "pages": pool,
                            "cache_bytes": kvp.cache_bytes, "contiguous_cache_bytes": kv.cache_bytes,
                            "output_equal_to_contiguous": bool(torch.equal(out, out_p)),
                            "note": "block-table indirection, pages shuffled over the sequences"}
            kvp.close()
            del kvp, out_p
    del graph

    # ---- dense fp16 baseline ----
    if want_fp16:
        res["fp16_baseline"] = fp16_baseline(w, lens, q_all, kf, vf, seq, steps, warmup, world, dev, peak, ms_step)
        del kf, vf
        torch.cuda.empty_cache()

    if full and not args.no_diag:
        # ---- per-layer logit MAE (K only): Block-GTQ against uniform TQ-MSE at
        # the same average width, over a 1024-position window of sequence 0 ----
        M = min(1024, lens[0])
        qd = torch.stack([wl.queries(w, l, 0, torch.arange(M), tag=3, device=dev) for l in range(L)])
        kd = torch.stack([wl.keys(w, l, 0, 0, M, device=dev) for l in range(L)])
        mae_g = torch.zeros((L, HQ), dtype=torch.float64, device=dev)
        kv.logit_mae(0, 0, 0, qd, kd, mae_g, layer_count=L)
        torch.cuda.synchronize()
        host_overhead_hidden()
        e0.record()
        kv.logit_mae(0, 0, 0, qd, kd, mae_g, layer_count=L)
        e1.record()
        torch.cuda.synchronize()
        diag_ms = e0.elapsed_time(e1)
        ucfg = bgtq.Config(**dict(wl.bench_config_fields(w), capacity_tokens=M, max_batch=1))
        kvu = bgtq.PackedKVCache(ucfg, dev)
        kvu.set_allocation(np.full((L, H, 64), w.k_bits, dtype=np.int8))
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        cnt = torch.full((1,), M, dtype=torch.int32, device=dev)
        kvu.encode_append(0, kd[:, None], kd[:, None], zero, cnt, layer_count=L)
        mae_u = torch.zeros((L, HQ), dtype=torch.float64, device=dev)
        kvu.logit_mae(0, 0, 0, qd, kd, mae_u, layer_count=L)
        torch.cuda.synchronize()
        assert kv.device_error() == 0 and kvu.device_error() == 0, "device error in the logit-MAE diagnostic"
        kvu.close()
        g_l = mae_g.mean(dim=1).cpu().numpy()
        u_l = mae_u.mean(dim=1).cpu().numpy()
        res["logit_mae"] = {"window": M, "pairs_per_head": M * (M + 1) // 2, "block_gtq_mean": float(g_l.mean()),
                            "tq_mse_mean": float(u_l.mean()), "reduction": float(1 - g_l.mean() / u_l.mean()),
                            "wins": f"{int((g_l < u_l).sum())}/{L}", "ms_all_layers": diag_ms,
                            "per_layer_block_gtq": [round(float(x), 5) for x in g_l],
                            "per_layer_tq_mse": [round(float(x), 5) for x in u_l],
                            "note": "K-only logit MAE (q.k / sqrt(128)) over causal pairs, synthetic Q/K"}
        del qd, kd

    # ---- the fused RoPE + encode (K before RoPE), timed after every decode
    # measurement: it rewrites the first chunk of layer 0 ----
    n_r = min(chunk, lens[0])
    kk = torch.zeros((1, B, n_r, H, 128), dtype=torch.float16, device=dev)
    kk[0, 0] = wl.keys(w, 0, 0, 0, n_r, device=dev)
    st0 = torch.zeros(B, dtype=torch.int32, device=dev)
    c0 = torch.zeros(B, dtype=torch.int32, device=dev)
    c0[0] = n_r
    rope_ms, g_r, _ = time_graph(lambda: kv.encode_append(0, kk, kk, st0, c0, rope_base=w.rope_base), 5, 3)
    del g_r
    assert kv.device_error() == 0, "device error in the fused RoPE + encode"
    res["prefill_encode_rope_rows_per_s"] = n_r * H / (rope_ms * 1e-3)
    del kk
    kv.close()
    del kv, q_all, knew, vnew, out, seq
    torch.cuda.empty_cache()

    # ---- CPU oracle on a bounded sample ----
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_units = 6 if full else 2
        max_tokens = None if full else 16384
        res["cpu_baseline"], _ = oracle_baseline(w, lens, n_units, max_pairs=3 if full else 1,
                                                 max_tokens=max_tokens)
    return res


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from packed_decode_attention_b200 import workloads as wl

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w = wl.WORKLOADS[args.workload]
    if args.layers:
        w = wl.scaled(w, n_layers=args.layers)
    lens = wl.seq_lens(w)
    r = measure(w, args, dev, world, rank, full=True)

    sides = None
    if world == 1 and not args.no_side and not args.layers:
        sides = {}
        for name in SIDE_WORKLOADS:
            if name == args.workload:
                continue
            sw = wl.WORKLOADS[name]
            try:
                s = measure(sw, args, dev, 1, rank, full=False)
                s["config"] = workload_config(sw, wl.seq_lens(sw))
                sides[name] = s
            except Exception as e:  # keep the headline line even if a side workload fails
                sides[name] = {"error": f"{type(e).__name__}: {str(e)[:200]}"}
                torch.cuda.empty_cache()

    line = {
        "metric": "decode_tokens_per_s", "value": r["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16*f16+f32 (mma.sync: fp16 operands, fp32 accumulate)",
        "data": "synthetic", "config": workload_config(w, lens),
    }
    for k in ("step_hbm_gbs", "roofline", "e2e", "gpu_launches", "clocks", "decode_path", "decode_wave_ctas", "buffered",
              "multi_layer", "decode_call", "fp16_baseline", "logit_mae", "paged", "cpu_baseline", "allocate_ms",
              "prefill_encode_rows_per_s", "prefill_encode_call_rows", "prefill_encode_call_ms",
              "prefill_encode_rope_rows_per_s",
              "compression_vs_fp16"):
        if k in r:
            line[k] = r[k]
    line["workloads"] = sides
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
