"""Seeded synthetic workloads (inputs only; none of the method's arithmetic).

The pages measure on real models (Qwen2.5-3B-Instruct, Llama-3.1-8B-Instruct,
...) over NIAH / LongBench / AIME text; none of that is available here, so
the inputs are synthetic with the shapes of those models:

* keys: per (layer, KV head, RoPE block) a standard deviation drawn
  log-normal(0, s) (both dims of a block share it), entries N(0, sigma^2),
  then RoPE at their cache positions, then fp16;
* values: N(0, 1) fp16;
* queries (calibration rows and the decode query): their own log-normal
  profile per (layer, KV head), shared by the G query heads of the group,
  independent rows per head, RoPE at positions 0..N-1 (calibration) and at
  the decode position; fp16;
* calibration keys: the first N_calib cached keys of sequence 0.

Named workloads (sizes of the five benchmark shapes):
  tiny    1 layer, 1 KV head, 4 q heads, 4096 tokens, K3V3, base 1e4, s = 1,  256 calib rows
  llama   1 layer, 8 KV heads, 32 q heads, 32768 tokens, K2V2, base 5e5, s = 1.5, 2048 calib rows
  qwen3b  36 layers, 2 KV heads, 16 q heads, 131072 tokens, K3V3, base 1e6, s = 1
  batch   28 layers, 4 KV heads, 28 q heads, 16 sequences of U[16384, 32768] tokens, K3V2, base 1e6, s = 1
  long    36 layers, 2 KV heads, 16 q heads, 524288 tokens, K3V3, base 1e6, s = 1 (+ a 131072-token encode chunk)
"""
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    batch: int
    seq_len: int            # cached tokens (the capacity for ragged batches)
    k_bits: int
    v_bits: int
    rope_base: float
    sigma: float            # log-normal shape of the per-block stds
    n_calib: int
    ragged: tuple = None    # (lo, hi) inclusive lengths, or None
    encode_chunk: int = 0   # rows of the timed prefill encode (long context)
    seed: int = 0

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 1, 4096, 3, 3, 1e4, 1.0, 256, seed=1001),
    "llama": Workload("llama", 1, 8, 32, 1, 32768, 2, 2, 5e5, 1.5, 2048, seed=1002),
    "qwen3b": Workload("qwen3b", 36, 2, 16, 1, 131072, 3, 3, 1e6, 1.0, 2048, seed=1003),
    "batch": Workload("batch", 28, 4, 28, 16, 32768, 3, 2, 1e6, 1.0, 2048, ragged=(16384, 32768), seed=1004),
    "long": Workload("long", 36, 2, 16, 1, 524288, 3, 3, 1e6, 1.0, 2048, encode_chunk=131072, seed=1005),
}


def _gen(w, *tags, device="cpu"):
    """A torch.Generator seeded from the workload seed and integer tags."""
    s = w.seed
    for t in tags:
        s = (s * 1000003 + int(t) + 7) % (2 ** 62)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def rope(x, positions, base, pairing=0):
    """Apply RoPE to x [..., T, H, 128] (float32) at integer positions [T]."""
    d = x.shape[-1]
    half = d // 2
    pos = torch.as_tensor(positions, dtype=torch.float64, device=x.device)
    inv = base ** (-torch.arange(half, dtype=torch.float64, device=x.device) * 2.0 / d)
    ang = pos[:, None] * inv[None, :]
    c = torch.cos(ang).to(torch.float32)[:, None, :]
    s = torch.sin(ang).to(torch.float32)[:, None, :]
    if pairing == 0:
        a, b = x[..., :half], x[..., half:]
        return torch.cat([a * c - b * s, a * s + b * c], dim=-1)
    a, b = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def block_stds(w, layer, kind, device="cpu"):
    """Per (KV head, block) stds [Hkv, 64]; kind 0 = keys, 1 = queries."""
    g = _gen(w, 11, layer, kind, device=device)
    z = torch.randn((w.n_kv_heads, 64), generator=g, device=device, dtype=torch.float32)
    return torch.exp(w.sigma * z)


def _expand(stds, pairing=0):
    """[H, 64] block stds -> [H, 128] dim stds."""
    if pairing == 0:
        return torch.cat([stds, stds], dim=-1)
    return stds.repeat_interleave(2, dim=-1)


def keys(w, layer, seq, start, count, device="cpu", pairing=0):
    """fp16 keys [count, Hkv, 128] of sequence ``seq`` at positions start..start+count-1."""
    sd = _expand(block_stds(w, layer, 0, device), pairing)
    g = _gen(w, 21, layer, seq, start, device=device)
    x = torch.randn((count, w.n_kv_heads, 128), generator=g, device=device, dtype=torch.float32) * sd
    return rope(x, torch.arange(start, start + count), w.rope_base, pairing).to(torch.float16)


def values(w, layer, seq, start, count, device="cpu"):
    g = _gen(w, 31, layer, seq, start, device=device)
    return torch.randn((count, w.n_kv_heads, 128), generator=g, device=device, dtype=torch.float32).to(torch.float16)


def queries(w, layer, seq, positions, tag=0, device="cpu", pairing=0):
    """fp16 queries [len(positions), Hq, 128]; the G heads of a group share the profile."""
    sd = _expand(block_stds(w, layer, 1, device), pairing).repeat_interleave(w.group, dim=0)
    pos = torch.as_tensor(positions)
    g = _gen(w, 41, layer, seq, tag, int(pos[0]) if len(pos) else 0, device=device)
    x = torch.randn((len(pos), w.n_q_heads, 128), generator=g, device=device, dtype=torch.float32) * sd
    return rope(x, pos, w.rope_base, pairing).to(torch.float16)


def calibration(w, device="cpu", pairing=0):
    """(calib_q [L, N, Hq, 128], calib_k [L, N, Hkv, 128]) fp16."""
    n = w.n_calib
    cq = torch.stack([queries(w, l, 0, torch.arange(n), tag=1, device=device, pairing=pairing)
                      for l in range(w.n_layers)])
    ck = torch.stack([keys(w, l, 0, 0, n, device=device, pairing=pairing) for l in range(w.n_layers)])
    return cq, ck


def seq_lens(w):
    """Cached lengths per sequence (int list)."""
    if w.ragged is None:
        return [w.seq_len] * w.batch
    rng = np.random.default_rng(w.seed)
    lo, hi = w.ragged
    return [int(x) for x in rng.integers(lo, hi + 1, size=w.batch)]


def decode_query(w, layer, lens, device="cpu", pairing=0):
    """fp16 [batch, Hq, 128]: each sequence's query at its decode position (= its length)."""
    return torch.stack([queries(w, layer, b, torch.tensor([lens[b]]), tag=2, device=device, pairing=pairing)[0]
                        for b in range(w.batch)])


def scaled(w, **changes):
    """A copy of the workload with some fields changed (smaller test cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)


def bench_config_fields(w):
    """Library config fields the benchmark and its full-size tests use for a workload."""
    return dict(n_layers=w.n_layers, n_kv_heads=w.n_kv_heads, n_q_heads=w.n_q_heads, max_batch=w.batch,
                capacity_tokens=w.seq_len, k_avg_bits=w.k_bits, v_avg_bits=w.v_bits, seed=w.seed,
                max_splits=64 if w.batch > 4 else 0)


def prefill(kv, w, lens, device, chunk=32768, on_chunk=None):
    """Append every sequence's keys/values [0, len) of every layer to a
    library cache, in chunks generated on ``device``.  ``on_chunk(layer, seq,
    start, k, v)`` sees each chunk (fp16 [n, Hkv, 128]) after it is queued."""
    for layer in range(w.n_layers):
        for b in range(w.batch):
            for s0 in range(0, lens[b], chunk):
                n = min(chunk, lens[b] - s0)
                kk = torch.zeros((1, w.batch, n, w.n_kv_heads, 128), dtype=torch.float16, device=device)
                vv = torch.zeros_like(kk)
                kk[0, b] = keys(w, layer, b, s0, n, device=device)
                vv[0, b] = values(w, layer, b, s0, n, device=device)
                start = torch.zeros(w.batch, dtype=torch.int32, device=device)
                count = torch.zeros(w.batch, dtype=torch.int32, device=device)
                start[b] = s0
                count[b] = n
                kv.encode_append(layer, kk, vv, start, count)
                if on_chunk is not None:
                    on_chunk(layer, b, s0, kk[0, b], vv[0, b])
