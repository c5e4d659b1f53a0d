"""The synthetic input generator: shapes, determinism, the stated distributions."""
import numpy as np
import torch

from packed_decode_attention_b200 import workloads as wl


def test_named_workloads_have_the_benchmark_shapes():
    w = wl.WORKLOADS
    assert (w["tiny"].n_kv_heads, w["tiny"].n_q_heads, w["tiny"].seq_len, w["tiny"].k_bits) == (1, 4, 4096, 3)
    assert (w["llama"].n_kv_heads, w["llama"].group, w["llama"].seq_len, w["llama"].k_bits) == (8, 4, 32768, 2)
    assert (w["qwen3b"].n_layers, w["qwen3b"].n_kv_heads, w["qwen3b"].group, w["qwen3b"].seq_len) == (36, 2, 8, 131072)
    assert (w["batch"].batch, w["batch"].group, w["batch"].v_bits) == (16, 7, 2)
    assert (w["long"].seq_len, w["long"].encode_chunk) == (524288, 131072)
    lens = wl.seq_lens(w["batch"])
    assert len(lens) == 16 and min(lens) >= 16384 and max(lens) <= 32768
    assert lens == wl.seq_lens(w["batch"])


def test_generator_is_deterministic_and_shaped():
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=64)
    a = wl.keys(w, 0, 0, 0, 64)
    b = wl.keys(w, 0, 0, 0, 64)
    assert a.dtype == torch.float16 and a.shape == (64, 1, 128)
    assert torch.equal(a, b)
    assert not torch.equal(a, wl.keys(w, 0, 0, 64, 64))
    cq, ck = wl.calibration(w)
    assert cq.shape == (1, 256, 4, 128) and ck.shape == (1, 256, 1, 128)
    q = wl.decode_query(w, 0, [64])
    assert q.shape == (1, 4, 128)


def test_key_block_energies_follow_the_lognormal_profile():
    """Per-block key energy is invariant under RoPE and tracks the drawn stds."""
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=4096)
    k = wl.keys(w, 0, 0, 0, 4096).float()[:, 0]
    e = (k[:, :64] ** 2 + k[:, 64:] ** 2).mean(0)
    sd = wl.block_stds(w, 0, 0)[0]
    assert torch.allclose(e, 2 * sd ** 2, rtol=0.15)
    v = wl.values(w, 0, 0, 0, 4096).float()
    assert abs(v.mean().item()) < 0.02 and abs(v.std().item() - 1) < 0.02


def test_rope_pairings_rotate_each_block():
    x = torch.randn(5, 2, 128)
    for pairing in (0, 1):
        y = wl.rope(x, torch.arange(100, 105), 1e4, pairing)
        if pairing == 0:
            nx = x[..., :64] ** 2 + x[..., 64:] ** 2
            ny = y[..., :64] ** 2 + y[..., 64:] ** 2
        else:
            nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
            ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
        assert torch.allclose(nx, ny, rtol=1e-5, atol=1e-5)
    assert torch.allclose(wl.rope(x, torch.zeros(5, dtype=torch.long), 1e4), x)
