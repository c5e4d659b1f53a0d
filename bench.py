#!/usr/bin/env python
"""Decode-attention throughput of the packed Block-GTQ cache on B200.

One step = one decode step of the whole model: for every layer, append the
step's new token to the packed cache (TQ-MSE encode of its K and V rows at
position len-1, so lengths stay fixed) and run GQA decode attention over the
packed cache (rotate the query, split-K pass, combine).  Steps run as one
CUDA graph.  value = sequences * steps / time  (decode tokens/s).

Printed as one JSON line on rank 0.  Also measured in the same run:
  roofline      the split-K decode kernel: its per-layer launches back to back
                in a captured graph (launch_ms) and with events around each
                launch (launch_ms_isolated), against the measured HBM peak
  e2e           same step through the C ABI from pinned host buffers (H2D of
                the queries and new K/V, D2H of the outputs inside the timing)
  multi_layer   all layers in one launch per kernel
  buffered      the step with 4 fp16 sink rows and a 128-row fp16 window
  paged         the step on a paged copy of the cache (shuffled pages)
  logit_mae     per-layer logit MAE, Block-GTQ against uniform TQ-MSE
  fp16_baseline dense fp16 FlashAttention-2 decode over the unquantised K/V
  cpu_baseline  the CPU oracle on a bounded sample (rank 0, one GPU)

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen3b]
  python bench.py --impl reference ...   (the CPU oracle as the reference arm)
"""
import argparse
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

# DRAM bytes (read + write) per split-kernel launch from the ncu capture
# summarised in profiles/decode_split_mma_qwen3b.md, for the workload it was
# taken on (an 8-layer copy of it: the same per-layer launch).  Reported as
# the roofline's "traffic"; None for other workloads.
NCU_TRAFFIC_PER_LAUNCH = {"qwen3b": 27.8839e6}


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


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        n = 1
    return max(n, 1)


class OracleSample:
    """A bounded sample of the workload for the CPU oracle: a few (layer, KV
    head) pairs of sequence 0 at its full length, each with its own oracle
    allocation, tables and packed cache (built once, untimed).  One timed unit
    is the oracle's decode of the G query heads of a pair over its cache plus
    the encode of one new K/V row; a full step is every (layer, KV head) of
    every sequence, so the step time is the unit time scaled by
    layers * KV heads * (total cached tokens / sample length)."""

    def __init__(self, w, lens, max_pairs=4):
        import numpy as np

        from oracle import model
        from packed_decode_attention_b200 import workloads as wl

        self.w, self.lens = w, lens
        pairs = [(l, h) for l in range(w.n_layers) for h in range(w.n_kv_heads)]
        self.n_pairs = len(pairs)
        pick = [pairs[i] for i in np.linspace(0, len(pairs) - 1, num=min(max_pairs, len(pairs))).astype(int)]
        self.t_len = lens[0]
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

    def time_unit(self, i):
        from oracle import model
        tb, l, h, k1, v1, q, enc = self.units[i % len(self.units)]
        t0 = time.perf_counter()
        model.encode_rows(tb, l, h, k1, v1)
        model.decode(tb, l, h, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], enc["n"])
        return time.perf_counter() - t0

    def step_seconds(self, unit_s):
        return unit_s * self.w.n_layers * self.w.n_kv_heads * (sum(self.lens) / float(self.t_len))

    def describe(self, n_timed):
        w = self.w
        return (f"oracle decode of the {w.group} query heads of one (layer, KV head) over {self.t_len} tokens "
                f"+ encode of one K/V row; {n_timed} units over {len(self.units)} of {self.n_pairs} pairs "
                f"(sequence 0 of {w.batch}); step time = unit time x {w.n_layers * w.n_kv_heads} pairs "
                f"x total/sample tokens")


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    from packed_decode_attention_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    lens = wl.seq_lens(w)
    sample = OracleSample(w, lens, max_pairs=2)
    times = []
    for i in range(args.warmup + args.steps):
        dt = sample.time_unit(i)
        if i >= args.warmup:
            times.append(sample.step_seconds(dt))
    step_s = statistics.mean(times)
    value = w.batch / step_s
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": "decode_tokens_per_s", "value": value, "unit": "tokens/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, lens),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample.describe(args.steps)},
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


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    from packed_decode_attention_b200 import bgtq
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
    L, H, HQ, B = w.n_layers, w.n_kv_heads, w.n_q_heads, w.batch
    cap = w.seq_len
    cfg = bgtq.Config(**wl.bench_config_fields(w))
    kv = bgtq.PackedKVCache(cfg, dev)
    stream = torch.cuda.current_stream()

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
    enc_ms = 0.0
    enc_rows = 0
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
                e0.record()
                kv.encode_append(l, kk, vv, start, count)
                e1.record()
                torch.cuda.synchronize()
                enc_ms += e0.elapsed_time(e1)
                enc_rows += n * H
    assert kv.device_error() == 0, "device error after prefill"

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
        # per layer: append the new K/V row, then attend (appends and query
        # rotation share one launch, then the split pass and the combine)
        for l in range(L):
            kv.decode_step(l, knew[l:l + 1], vnew[l:l + 1], start1, count1, q_all[l:l + 1], seq, out[l:l + 1])

    def step_multi():
        kv.encode_append(0, knew, vnew, start1, count1, layer_count=L)
        kv.decode_attn(0, q_all, seq, out, layer_count=L)

    def time_graph(fn, steps, warmup, sampler=None):
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

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid, local)
    sampler.start()
    time.sleep(0.5)
    ms_step, graph, (tw0, tw1) = time_graph(step, args.steps, args.warmup)
    sampler.stop()
    clocks = sampler.summary(tw0, tw1)
    ms_step = max_over_ranks(ms_step, world, dev)
    assert kv.device_error() == 0, "device error during the timed steps"
    out_check = out.float()
    assert torch.isfinite(out_check).all(), "non-finite decode output"

    ms_multi, g_multi, _ = time_graph(step_multi, args.steps, args.warmup)
    ms_multi = max_over_ranks(ms_multi, world, dev)
    del g_multi

    # ---- the same step with an fp16 sink + recent window (the README's
    # "withbuffer" setting): packed positions [sink, len - window) plus the
    # buffered rows ----
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
            kv.decode_step_buffered(l, knew[l:l + 1], vnew[l:l + 1], start1, count1, q_all[l:l + 1], seq_hi, seq_lo,
                                    buf_k[l:l + 1], buf_v[l:l + 1], buf_cnt, out[l:l + 1])

    ms_buf, g_buf, _ = time_graph(step_buffered, args.steps, args.warmup)
    ms_buf = max_over_ranks(ms_buf, world, dev)
    del g_buf, buf_k, buf_v
    assert kv.device_error() == 0, "device error in the buffered step"

    # ---- the same step over a paged copy of the cache: a tight pool of
    # 64-position pages, shuffled over the sequences' tiles ----
    paged = None
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

        ms_paged, g_p, _ = time_graph(step_paged, args.steps, args.warmup)
        ms_paged = max_over_ranks(ms_paged, world, dev)
        del g_p
        step()
        step_paged()
        torch.cuda.synchronize()
        assert kvp.device_error() == 0, "device error in the paged step"
        paged = {"ms_per_step": ms_paged, "tokens_per_s": world * B / (ms_paged * 1e-3), "pages": pool,
                 "cache_bytes": kvp.cache_bytes, "contiguous_cache_bytes": kv.cache_bytes,
                 "output_equal_to_contiguous": bool(torch.equal(out, out_p)),
                 "note": "block-table indirection, pages shuffled over the sequences"}
        kvp.close()
        del kvp, out_p

    # ---- the split-K kernel in isolation: events around each per-layer
    # launch, in a captured step (the event nodes keep the split kernel from
    # overlapping its neighbours, so each interval is that kernel's whole
    # duration, start-up included) ----
    tb = token_bytes(kv, cfg)
    qrot = torch.empty((1, B, HQ, 128), dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(L)]

    def step_timed_split():
        for l in range(L):
            kv.encode_append(l, knew[l:l + 1], vnew[l:l + 1], start1, count1)
            kv.rotate_query(l, q_all[l:l + 1], qrot)
            ev[l][0].record()
            kv.decode_split(l, qrot, seq)
            ev[l][1].record()
            kv.decode_combine(l, seq, out[l:l + 1])

    step_timed_split()
    torch.cuda.synchronize()
    g_split = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_split):
        step_timed_split()
    split_ms = []
    for it in range(args.warmup + args.steps):
        g_split.replay()
        torch.cuda.synchronize()
        if it >= args.warmup:
            split_ms.extend(a.elapsed_time(z) for a, z in ev)
    del g_split
    split_isolated_ms = statistics.mean(split_ms)

    # ---- the split kernel's average launch duration: the step's per-layer
    # split launches (same inputs, same launch configuration) back to back in
    # one captured graph, CUDA events around the whole timed region, divided
    # by the launches; each launch's set-up overlaps the previous one's tail,
    # as in the step ----
    qrot_all = torch.empty((L, B, HQ, 128), dtype=torch.float32, device=dev)
    for l in range(L):
        kv.rotate_query(l, q_all[l:l + 1], qrot_all[l:l + 1])

    def splits_back_to_back():
        for l in range(L):
            kv.decode_split(l, qrot_all[l:l + 1], seq)

    ms_splits, g_sp, _ = time_graph(splits_back_to_back, args.steps, args.warmup)
    del g_sp
    split_avg_ms = max_over_ranks(ms_splits / L, world, dev)
    bytes_per_layer = [sum(lens[b] * tb[l, h] for b in range(B) for h in range(H)) for l in range(L)]
    alg_bytes = statistics.mean(bytes_per_layer)
    achieved = alg_bytes / (split_avg_ms * 1e-3) / 1e9
    peak, peak_kind = peaks()

    # ---- end to end from pinned host memory ----
    q_h = q_all.cpu().pin_memory()
    k_h = knew.cpu().pin_memory()
    v_h = vnew.cpu().pin_memory()
    o_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = q_h.numel() * 2 + k_h.numel() * 2 + v_h.numel() * 2
    d2h = o_h.numel() * 2
    for _ in range(args.warmup):
        q_all.copy_(q_h, non_blocking=True)
        knew.copy_(k_h, non_blocking=True)
        vnew.copy_(v_h, non_blocking=True)
        graph.replay()
        o_h.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        q_all.copy_(q_h, non_blocking=True)
        knew.copy_(k_h, non_blocking=True)
        vnew.copy_(v_h, non_blocking=True)
        graph.replay()
        o_h.copy_(out, non_blocking=True)
    z.record()
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(a.elapsed_time(z) / args.steps, world, dev)
    del graph

    # ---- dense fp16 baseline (FlashAttention-2 decode) ----
    fp16 = None
    if want_fp16:
        import torch.nn.functional as F
        qf = q_all.view(L, B, 1, HQ, 128)

        def fp16_step_sdpa():
            for l in range(L):
                for b in range(B):
                    qq = q_all[l, b][None, :, None, :]
                    kk = kf[l][b, :lens[b]].transpose(0, 1)[None]
                    vv = vf[l][b, :lens[b]].transpose(0, 1)[None]
                    F.scaled_dot_product_attention(qq, kk, vv, enable_gqa=True)

        try:
            from flash_attn import flash_attn_with_kvcache

            def fp16_step():
                for l in range(L):
                    flash_attn_with_kvcache(qf[l], kf[l], vf[l], cache_seqlens=seq)

            fp16_step()
            torch.cuda.synchronize()
            name = "flash_attn_with_kvcache (FlashAttention-2 decode)"
        except Exception:
            fp16_step = fp16_step_sdpa
            name = "torch scaled_dot_product_attention"
        try:
            ms_fp16, g16, _ = time_graph(fp16_step, args.steps, args.warmup)
            ms_fp16 = max_over_ranks(ms_fp16, world, dev)
            del g16
            fp16 = {"impl": name, "ms_per_step": ms_fp16, "tokens_per_s": world * B / (ms_fp16 * 1e-3),
                    "bytes_per_step": int(sum(lens) * H * L * 512), "speedup_of_packed": ms_fp16 / ms_step}
        except Exception as e:  # report, do not fail the bench
            fp16 = {"impl": name, "error": str(e)[:200]}
        del kf, vf

    # ---- per-layer logit MAE (K only): Block-GTQ against uniform TQ-MSE at
    # the same average width, over a 1024-position window of sequence 0 ----
    diag = None
    if not args.no_diag:
        M = min(1024, lens[0])
        qd = torch.stack([wl.queries(w, l, 0, torch.arange(M), tag=3, device=dev) for l in range(L)])
        kd = torch.stack([wl.keys(w, l, 0, 0, M, device=dev) for l in range(L)])
        mae_g = torch.zeros((L, HQ), dtype=torch.float64, device=dev)
        kv.logit_mae(0, 0, 0, qd, kd, mae_g, layer_count=L)
        torch.cuda.synchronize()
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
        diag = {"window": M, "pairs_per_head": M * (M + 1) // 2, "block_gtq_mean": float(g_l.mean()),
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
    rope_ms = []
    for it in range(4):
        e0.record()
        kv.encode_append(0, kk, kk, st0, c0, rope_base=w.rope_base)
        e1.record()
        torch.cuda.synchronize()
        if it:
            rope_ms.append(e0.elapsed_time(e1))
    assert kv.device_error() == 0, "device error in the fused RoPE + encode"
    rope_rows_per_s = n_r * H / (statistics.mean(rope_ms) * 1e-3)
    del kk

    # ---- CPU oracle on a bounded sample ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(w, lens, max_pairs=3)
        units = [sample.time_unit(i) for i in range(len(sample.units) * 2)]
        st = sample.step_seconds(statistics.mean(units))
        cpu = {"value": B / st, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample.describe(len(units))}

    value = job_value(world, B, ms_step)
    step_bytes = sum(bytes_per_layer) + L * B * HQ * 512
    line = {
        "metric": "decode_tokens_per_s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, lens),
        "step_hbm_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": NCU_TRAFFIC_PER_LAUNCH.get(args.workload), "kernel": "decode_mma_kernel",
                     "launch_ms": split_avg_ms, "alg_bytes_per_launch": alg_bytes, "peak_kind": peak_kind,
                     "launch_ms_isolated": split_isolated_ms,
                     "timing": "launch_ms: the step's per-layer split launches back to back in a captured graph, "
                               "events around the region / launches; launch_ms_isolated: events around each "
                               "launch inside a captured step (start-up not overlapped)"},
        "e2e": {"value": world * B / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * L * args.steps,
        "clocks": clocks,
        "buffered": {"ms_per_step": ms_buf, "tokens_per_s": world * B / (ms_buf * 1e-3), "sink": SINK,
                     "window": WINDOW, "note": "fp16 sink + recent window next to the packed cache"},
        "multi_layer": {"ms_per_step": ms_multi, "tokens_per_s": world * B / (ms_multi * 1e-3),
                        "hbm_gbs": step_bytes / (ms_multi * 1e-3) / 1e9},
        "fp16_baseline": fp16,
        "logit_mae": diag,
        "paged": paged,
        "cpu_baseline": cpu,
        "allocate_ms": alloc_ms,
        "prefill_encode_rows_per_s": enc_rows / (enc_ms * 1e-3),
        "prefill_encode_call_rows": chunk,
        "prefill_encode_rope_rows_per_s": rope_rows_per_s,
        "compression_vs_fp16": 512.0 / (sum(lens[b] * tb[l, h] for l in range(L) for b in range(B) for h in range(H))
                                        / (sum(lens) * L * H)),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    kv.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
