"""GPU parity of the per-layer logit MAE (Block-GTQ abstract: logit fidelity
per layer; blockgtq README, bit allocation: per-layer kernel MAE against
uniform TQ-MSE) against the oracle, on identical packed caches (the oracle's
tiles uploaded into the library)."""
import numpy as np
import pytest
import torch

from oracle import diag, model
from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl
from parity_helpers import encode_on_gpu, library_config, oracle_config, upload_oracle_rows

pytestmark = pytest.mark.gpu

MAE_REL_TOL = 1e-4   # fp32 logits of both sides; an off-by-one in the causal mask moves the MAE by ~2 / M


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda:0")


@pytest.mark.parametrize("n_kv,n_q,m,w0,seq,layers", [
    (1, 4, 200, 0, 0, 1),      # one KV head, G = 4, aligned window
    (2, 16, 130, 37, 1, 2),    # G = 8, window starting inside a tile, second sequence, two layers per call
    (2, 14, 65, 64, 0, 1),     # G = 7 (the batch workload's group)
    (1, 12, 100, 5, 0, 1),     # G = 12: two blocks of query heads
    (1, 4, 1, 70, 0, 1),       # a single pair
])
def test_logit_mae_matches_oracle(dev, n_kv, n_q, m, w0, seq, layers):
    w = wl.scaled(wl.WORKLOADS["tiny"], n_layers=layers, n_kv_heads=n_kv, n_q_heads=n_q, batch=seq + 1,
                  seq_len=w0 + m, n_calib=64)
    cfg = library_config(w)
    kv = bgtq.PackedKVCache(cfg, dev)
    cq, ck = wl.calibration(w)
    ocfg = oracle_config(cfg)
    widths = model.allocate(ocfg, cq.numpy(), ck.numpy())
    kv.set_allocation(widths.astype(np.int8))
    tb = model.Tables(ocfg, widths)
    g = cfg.group_size
    qs, ks, want = [], [], np.zeros((layers, n_q))
    for layer in range(layers):
        k = wl.keys(w, layer, seq, 0, w0 + m)
        q = wl.queries(w, layer, seq, torch.arange(w0, w0 + m), tag=3)
        qs.append(q)
        ks.append(k[w0:])
        for h in range(n_kv):
            enc = model.encode_rows(tb, layer, h, k[:, h].numpy(), k[:, h].numpy())
            upload_oracle_rows(kv, layer, seq, h, enc)
            want[layer, h * g:(h + 1) * g] = diag.logit_mae(tb, layer, h, q[:, h * g:(h + 1) * g].numpy(),
                                                            k[w0:, h].numpy(), enc["k_tiles"], enc["k_norms"], w0)
    out = torch.full((layers, n_q), float("nan"), dtype=torch.float64, device=dev)
    kv.logit_mae(0, seq, w0, torch.stack(qs).to(dev), torch.stack(ks).to(dev), out, layer_count=layers)
    torch.cuda.synchronize()
    assert kv.device_error() == 0
    got = out.cpu().numpy()
    np.testing.assert_allclose(got, want, rtol=MAE_REL_TOL, atol=0)
    kv.close()


def test_block_gtq_beats_uniform_every_layer(dev):
    """The pages' per-layer comparison in synthetic form, through the
    library alone: the qwen3b shape (8 of its layers), a 1024-position
    window, Block-GTQ allocated on the GPU from calibration rows against
    uniform 3-bit TQ-MSE, both encoding the same keys."""
    w = wl.scaled(wl.WORKLOADS["qwen3b"], n_layers=8, seq_len=1024, n_calib=1024)
    m = 1024
    cq, ck = wl.calibration(w, device=dev)
    res = []
    for mode in ("gtq", "uniform"):
        cfg = library_config(w)
        kv = bgtq.PackedKVCache(cfg, dev)
        if mode == "gtq":
            kv.allocate(cq, ck)
        else:
            kv.set_allocation(np.full((w.n_layers, w.n_kv_heads, 64), 3, dtype=np.int8))
        encode_on_gpu(kv, w, range(w.n_layers), [m], dev)
        q = torch.stack([wl.queries(w, l, 0, torch.arange(m), tag=3, device=dev) for l in range(w.n_layers)])
        k = torch.stack([wl.keys(w, l, 0, 0, m, device=dev) for l in range(w.n_layers)])
        out = torch.zeros((w.n_layers, w.n_q_heads), dtype=torch.float64, device=dev)
        kv.logit_mae(0, 0, 0, q, k, out, layer_count=w.n_layers)
        torch.cuda.synchronize()
        assert kv.device_error() == 0
        res.append(out.mean(dim=1).cpu().numpy())
        kv.close()
    gtq, uni = res
    assert np.all(np.isfinite(gtq)) and np.all(gtq > 0)
    assert np.all(gtq < uni), (gtq, uni)


def test_logit_mae_rejects_bad_windows(dev):
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=256, n_calib=64)
    kv = bgtq.PackedKVCache(library_config(w), dev)
    kv.set_allocation(np.full((1, 1, 64), 3, dtype=np.int8))
    q = torch.zeros((1, 200, 4, 128), dtype=torch.float16, device=dev)
    k = torch.zeros((1, 200, 1, 128), dtype=torch.float16, device=dev)
    out = torch.zeros((1, 4), dtype=torch.float64, device=dev)
    for seq, w0 in [(0, 57), (1, 0), (0, -1)]:   # past capacity, no such sequence, negative start
        with pytest.raises(bgtq.BgtqError):
            kv.logit_mae(0, seq, w0, q, k, out)
    kv.close()
