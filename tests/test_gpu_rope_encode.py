"""The fused RoPE + encode (bgtq_encode_append_rope) against the oracle's
fused encode: K rows taken before RoPE, turned at their cache positions and
encoded.  Both kernels (a prefill call and a call of at most 16 rows per
sequence), both RoPE pairings, unaligned starts at large positions."""
import numpy as np
import pytest
import torch

from oracle import model, rope, tiles, tqmse
from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl
from parity_helpers import CODE_AGREEMENT, compare_codes, fp16_ulp_apart, library_config, oracle_config

pytestmark = pytest.mark.gpu

BASE = 1e6


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda:0")


def _codes_agree(frac, ok, nbad):
    """At least CODE_AGREEMENT of the codes equal (or a single mismatch in a
    small sample), every mismatch one code apart within the threshold slack."""
    return ok and (frac >= CODE_AGREEMENT or nbad <= 1)


def _pre_rope_rows(rows, heads, seed):
    g = torch.Generator().manual_seed(seed)
    std = torch.exp(torch.randn((heads, 128), generator=g))
    return (torch.randn((rows, heads, 128), generator=g) * std).half()


@pytest.mark.parametrize("pairing", [0, 1])
@pytest.mark.parametrize("rows,p0", [(300, 524261), (13, 131011), (1, 64)])
def test_fused_encode_matches_oracle(dev, pairing, rows, p0):
    w = wl.scaled(wl.WORKLOADS["tiny"], n_kv_heads=2, n_q_heads=8, seq_len=p0 + rows + 64, n_calib=128)
    cfg = library_config(w, rope_pairing=pairing)
    ocfg = oracle_config(cfg)
    cq, ck = wl.calibration(w, pairing=pairing)
    widths = model.allocate(ocfg, cq.numpy(), ck.numpy())
    kv = bgtq.PackedKVCache(cfg, dev)
    kv.set_allocation(widths.astype(np.int8))
    tb = model.Tables(ocfg, widths)
    k = _pre_rope_rows(rows, w.n_kv_heads, 11 + rows)
    v = _pre_rope_rows(rows, w.n_kv_heads, 12 + rows)
    one = torch.ones(1, dtype=torch.int32, device=dev)
    kv.encode_append(0, k[None, None].to(dev), v[None, None].to(dev), one * p0, one * rows, rope_base=BASE)
    torch.cuda.synchronize()
    assert kv.device_error() == 0
    pos = np.arange(p0, p0 + rows)
    t0, t1 = p0 // 64, (p0 + rows + 63) // 64
    off = p0 - 64 * t0
    for h in range(w.n_kv_heads):
        enc = model.encode_rows_rope(tb, 0, h, k[:, h].numpy(), v[:, h].numpy(), pos, BASE)
        groups = tb.groups[0, h]
        kt = kv.k_tiles()[0, 0, h, t0:t1].cpu().numpy()
        vt = kv.v_tiles()[0, 0, h, t0:t1].cpu().numpy()
        g_k = tiles.unpack_k_tiles(kt, groups, 64 * (t1 - t0))[off:off + rows]
        g_v = tiles.unpack_v_tiles(vt, cfg.v_avg_bits, 64 * (t1 - t0))[off:off + rows]
        # the oracle's u of the turned rows (float64, not rounded)
        x = rope.apply_rope(k[:, h].numpy().astype(np.float64), pos, BASE, pairing)
        u = np.concatenate([tqmse.rotated_normalised(x, dims, tb.k_rot[0, h][b])[0] for b, dims in groups], axis=1)
        frac, ok, nbad = compare_codes(g_k, enc["k_codes"], u, tqmse.record_widths(groups))
        assert _codes_agree(frac, ok, nbad), (h, frac, nbad)
        # values are not turned: the plain encode's bars
        uv = tqmse.rotated_normalised(v[:, h].numpy().astype(np.float64), np.arange(128), tb.v_rot[0, h])[0]
        frac, ok, nbad = compare_codes(g_v, enc["v_codes"], uv, np.full(128, cfg.v_avg_bits))
        assert _codes_agree(frac, ok, nbad), (h, frac, nbad)
        kn = kv.k_norms()[0, 0, h, p0:p0 + rows].cpu().numpy()
        assert np.all(fp16_ulp_apart(kn, enc["k_norms"]) <= 1), h
        vn = kv.v_norms()[0, 0, h, p0:p0 + rows].cpu().numpy()
        assert np.all(fp16_ulp_apart(vn, enc["v_norm"]) <= 1), h
    kv.close()


def test_fused_encode_rejects_bad_bases(dev):
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=256, n_calib=16)
    kv = bgtq.PackedKVCache(library_config(w), dev)
    kv.set_allocation(np.full((1, 1, 64), 3, dtype=np.int8))
    k = torch.zeros((1, 1, 4, 1, 128), dtype=torch.float16, device=dev)
    one = torch.ones(1, dtype=torch.int32, device=dev)
    for base in (1.0, 0.5, float("nan"), float("inf"), -1e4):
        with pytest.raises(bgtq.BgtqError) as e:
            kv.encode_append(0, k, k, one, one, rope_base=base)
        assert e.value.status == -1
    kv.close()
