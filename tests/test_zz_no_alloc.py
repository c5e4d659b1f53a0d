"""The static-scratch decode entry point, for callers that cannot allocate
device memory (stream-capture regions, runtimes whose device memory is all
reserved by their own pool): bgtq_decode_attn_static_scratch keeps its
split-K scratch in the library's own static device array.  Its output must
match bgtq_decode_attn within the decode tolerance, on consecutive calls
(the array keeps the previous call's contents).  Collected last on purpose."""
import numpy as np
import pytest
import torch

from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl

from parity_helpers import REL_TOL, library_config, row_rel_err

pytestmark = pytest.mark.gpu


def _filled_cache(w, dev, lens):
    cfg = library_config(w)
    kv = bgtq.PackedKVCache(cfg, dev)
    cq, ck = wl.calibration(w)
    kv.allocate(cq.to(dev), ck.to(dev))
    for l in range(w.n_layers):
        for b, ln in enumerate(lens):
            k = torch.zeros((1, w.batch, ln, w.n_kv_heads, 128), dtype=torch.float16)
            v = torch.zeros_like(k)
            k[0, b] = wl.keys(w, l, b, 0, ln)
            v[0, b] = wl.values(w, l, b, 0, ln)
            start = torch.zeros(w.batch, dtype=torch.int32, device=dev)
            count = torch.zeros(w.batch, dtype=torch.int32, device=dev)
            count[b] = ln
            kv.encode_append(l, k.to(dev), v.to(dev), start, count)
    return cfg, kv


@pytest.mark.parametrize("path", [0, 1])
def test_static_scratch_decode_matches_decode_attn_twice(path):
    """path 0: the three-launch decode; 1: the fused launch (both keep their
    scratch in the static array)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    dev = torch.device("cuda:0")
    w = wl.scaled(wl.WORKLOADS["llama"], n_layers=2, n_kv_heads=4, n_q_heads=16, batch=2, seq_len=3000,
                  n_calib=128)
    lens = [3000, 1234]
    cfg, kv = _filled_cache(w, dev, lens)
    kv.set_decode_path(path)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    for call, layer in enumerate((0, 1)):
        q = wl.decode_query(w, layer, lens)[None].to(dev)
        ref = torch.empty((1, 2, cfg.n_q_heads, 128), dtype=torch.float16, device=dev)
        kv.decode_attn(layer, q, seq, ref)
        got = torch.full_like(ref, float("nan"))
        bgtq.bgtq_decode_attn_static_scratch(kv.state, layer, 1, q, seq, 2, got)
        torch.cuda.synchronize()
        err = row_rel_err(got[0].float().cpu().numpy(), ref[0].float().cpu().numpy())
        assert np.all(err <= REL_TOL), (call, err.max())
    # both layers in one call also fit the static array
    q2 = torch.stack([wl.decode_query(w, l, lens) for l in range(2)]).to(dev)
    ref2 = torch.empty((2, 2, cfg.n_q_heads, 128), dtype=torch.float16, device=dev)
    kv.decode_attn(0, q2, seq, ref2, layer_count=2)
    got2 = torch.full_like(ref2, float("nan"))
    bgtq.bgtq_decode_attn_static_scratch(kv.state, 0, 2, q2, seq, 2, got2)
    torch.cuda.synchronize()
    assert np.all(row_rel_err(got2.float().cpu().numpy(), ref2.float().cpu().numpy()) <= REL_TOL)
    assert kv.device_error() == 0
    kv.close()


def test_static_scratch_rejects_oversized_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    dev = torch.device("cuda:0")
    # 8 sequences x 32 heads x 1024 splits of 528 bytes is far beyond 16 MiB
    cfg = bgtq.Config(n_layers=1, n_kv_heads=8, n_q_heads=32, max_batch=8, capacity_tokens=1 << 18,
                      max_splits=1024)
    kv = bgtq.PackedKVCache(cfg, dev)
    kv.set_allocation(np.full((1, 8, 64), 3, dtype=np.int8))
    kv.set_split_tokens(256)
    q = torch.zeros((1, 8, 32, 128), dtype=torch.float16, device=dev)
    seq = torch.ones(8, dtype=torch.int32, device=dev)
    out = torch.zeros_like(q)
    with pytest.raises(bgtq.BgtqError) as e:
        bgtq.bgtq_decode_attn_static_scratch(kv.state, 0, 1, q, seq, 8, out)
    assert e.value.status == -4
    kv.close()
