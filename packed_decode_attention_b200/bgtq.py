"""Python binding of the C ABI in include/bgtq.h (ctypes, argument marshalling only).

Every ``bgtq_*`` function here calls the function of the same name in the
in-tree ``libbgtq.so``; nothing is computed in Python.  ``PackedKVCache``
owns the two device buffers (torch tensors) and one library state.

The library must be built (``python -m packed_decode_attention_b200.build``
or ``__graft_entry__.build()``); importing the binding without it raises.

A decode step, per layer ``l`` (tensors on the GPU; shapes in include/bgtq.h)::

    kv = PackedKVCache(Config(n_layers=36, n_kv_heads=2, n_q_heads=16,
                              max_batch=1, capacity_tokens=131072), "cuda")
    kv.allocate(calib_q, calib_k)                    # Block-GTQ widths + tables
    kv.encode_append(l, k, v, start, count)          # prefill
    kv.decode_step(l, k_new, v_new, start, count,    # append the new rows,
                   q, seq_lens, out)                 # then attend
"""
import ctypes
import os
from dataclasses import dataclass, fields

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbgtq.so")

HEAD_DIM = 128
N_BLOCKS = HEAD_DIM // 2
TILE = 64

DEVERR_CAPACITY = 1
DEVERR_SEQ_LEN = 2
DEVERR_ARG = 4
DEVERR_NONFINITE = 8
DEVERR_TIMEOUT = 16
DEVERR_PAGE = 32


class BgtqError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"bgtq status {status}: {message}")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("max_batch", ctypes.c_int32),
        ("k_avg_bits", ctypes.c_int32),
        ("v_avg_bits", ctypes.c_int32),
        ("b_min", ctypes.c_int32),
        ("b_max", ctypes.c_int32),
        ("rope_pairing", ctypes.c_int32),
        ("max_splits", ctypes.c_int32),
        ("page_pool_tiles", ctypes.c_int32),
        ("capacity_tokens", ctypes.c_int64),
        ("seed", ctypes.c_uint64),
    ]


@dataclass
class Config:
    """Mirror of bgtq_config."""
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    max_batch: int
    capacity_tokens: int
    k_avg_bits: int = 3
    v_avg_bits: int = 3
    b_min: int = 1
    b_max: int = 4
    rope_pairing: int = 0
    max_splits: int = 0
    seed: int = 0
    head_dim: int = HEAD_DIM
    page_pool_tiles: int = 0   # > 0: paged cache (pages per layer and KV head)

    def to_c(self):
        c = _Config()
        for f in fields(self):
            setattr(c, f.name, getattr(self, f.name))
        return c

    @property
    def group_size(self):
        return self.n_q_heads // self.n_kv_heads


_lib = None
_VP = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIGS = {
    "bgtq_required_bytes": (ctypes.c_int, [ctypes.POINTER(_Config), ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "bgtq_create": (ctypes.c_int, [ctypes.POINTER(_Config), _VP, ctypes.c_size_t, _VP, ctypes.c_size_t, _VP, ctypes.POINTER(_VP)]),
    "bgtq_destroy": (None, [_VP]),
    "bgtq_allocate": (ctypes.c_int, [_VP, _VP, _I32, _VP, _I32, _VP]),
    "bgtq_set_allocation": (ctypes.c_int, [_VP, _VP, _VP]),
    "bgtq_get_allocation": (ctypes.c_int, [_VP, _VP]),
    "bgtq_get_energy": (ctypes.c_int, [_VP, _VP, _VP]),
    "bgtq_get_codebook": (ctypes.c_int, [_I32, _VP, _VP]),
    "bgtq_get_layout": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _VP]),
    "bgtq_get_rotation": (ctypes.c_int, [_VP, _I32, _I32, _I32, _I32, _VP, _VP]),
    "bgtq_cache_offsets": (ctypes.c_int, [_VP, _VP]),
    "bgtq_encode_append": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _I32, _VP]),
    "bgtq_encode_append_rope": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _I32, ctypes.c_double,
                                               _VP]),
    "bgtq_rotate_query": (ctypes.c_int, [_VP, _I32, _I32, _VP, _I32, _VP, _VP]),
    "bgtq_decode_attn": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _I32, _VP, _VP]),
    "bgtq_decode_attn_buffered": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _I32, _VP, _VP, _VP, _I32, _VP, _VP]),
    "bgtq_logit_mae": (ctypes.c_int, [_VP, _I32, _I32, _I32, _I32, _I32, _VP, _VP, _VP, _VP]),
    "bgtq_decode_step": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _VP, _VP, _I32, _VP, _VP]),
    "bgtq_decode_step_buffered": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _VP, _VP, _VP, _I32, _VP,
                                                 _VP, _VP, _I32, _VP, _VP]),
    "bgtq_set_block_table": (ctypes.c_int, [_VP, _VP]),
    "bgtq_test_drop_tile_copies": (ctypes.c_int, [_VP, _I32]),
    "bgtq_decode_split": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _I32, _VP]),
    "bgtq_decode_combine": (ctypes.c_int, [_VP, _I32, _I32, _VP, _I32, _VP, _VP]),
    "bgtq_decode_attn_static_scratch": (ctypes.c_int, [_VP, _I32, _I32, _VP, _VP, _I32, _VP, _VP]),
    "bgtq_set_split_tokens": (ctypes.c_int, [_VP, _I32]),
    "bgtq_set_decode_path": (ctypes.c_int, [_VP, _I32]),
    "bgtq_get_decode_path": (ctypes.c_int, [_VP, _VP, _VP]),
    "bgtq_get_device_error": (ctypes.c_int, [_VP, _VP, _VP]),
    "bgtq_error_string": (ctypes.c_char_p, [_I32]),
}


def lib():
    """The loaded libbgtq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m packed_decode_attention_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def declared_symbols():
    return list(_SIGS)


def _check(status):
    if status != 0:
        raise BgtqError(status, lib().bgtq_error_string(status).decode())


def _ptr(x):
    """Device or host address of a torch tensor / numpy array / int."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


ERR_INVALID_ARG = -1


def _expect(t, name, shape, dtype, device):
    """Raises BgtqError(ERR_INVALID_ARG) unless t is a contiguous torch tensor
    of dtype on device with this shape (None: any extent).  PackedKVCache
    checks its tensors this way before a pointer reaches the library, which
    reads the layouts that include/bgtq.h states."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise BgtqError(ERR_INVALID_ARG, f"{name}: a torch tensor is expected")
    if t.dtype != dtype:
        raise BgtqError(ERR_INVALID_ARG, f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device.type != device.type or (device.index is not None and t.device.index != device.index):
        raise BgtqError(ERR_INVALID_ARG, f"{name}: on {t.device}, expected {device}")
    if t.dim() != len(shape) or any(e is not None and t.shape[i] != e for i, e in enumerate(shape)):
        want = tuple("*" if e is None else e for e in shape)
        raise BgtqError(ERR_INVALID_ARG, f"{name}: shape {tuple(t.shape)}, expected {want}")
    if not t.is_contiguous():
        raise BgtqError(ERR_INVALID_ARG, f"{name}: not contiguous")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ---- same-name wrappers -------------------------------------------------

def bgtq_required_bytes(cfg):
    c = cfg.to_c()
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().bgtq_required_bytes(ctypes.byref(c), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def bgtq_create(cfg, d_cache, cache_bytes, d_workspace, workspace_bytes, stream=None):
    c = cfg.to_c()
    out = _VP()
    _check(lib().bgtq_create(ctypes.byref(c), _ptr(d_cache), cache_bytes, _ptr(d_workspace), workspace_bytes,
                             _stream(stream), ctypes.byref(out)))
    return out.value


def bgtq_destroy(state):
    lib().bgtq_destroy(state)


def bgtq_allocate(state, d_calib_q, nq, d_calib_k, nk, stream=None):
    _check(lib().bgtq_allocate(state, _ptr(d_calib_q), nq, _ptr(d_calib_k), nk, _stream(stream)))


def bgtq_set_allocation(state, h_widths, stream=None):
    w = np.ascontiguousarray(h_widths, dtype=np.int8)
    _check(lib().bgtq_set_allocation(state, w.ctypes.data, _stream(stream)))


def bgtq_get_allocation(state, n_layers, n_kv_heads):
    w = np.zeros((n_layers, n_kv_heads, N_BLOCKS), dtype=np.int8)
    _check(lib().bgtq_get_allocation(state, w.ctypes.data))
    return w


def bgtq_get_energy(state, n_layers, n_kv_heads):
    """Exact energies as nested lists of Python ints [L][Hkv][64] (units 2**-48)."""
    eq = np.zeros((n_layers, n_kv_heads, N_BLOCKS, 2), dtype=np.uint64)
    ek = np.zeros_like(eq)
    _check(lib().bgtq_get_energy(state, eq.ctypes.data, ek.ctypes.data))
    to_int = lambda a: [[[int(a[l, h, j, 0]) + (int(a[l, h, j, 1]) << 64) for j in range(N_BLOCKS)]
                         for h in range(n_kv_heads)] for l in range(n_layers)]
    return to_int(eq), to_int(ek)


def bgtq_get_codebook(bits):
    c = np.zeros(1 << bits, dtype=np.float32)
    t = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check(lib().bgtq_get_codebook(bits, c.ctypes.data, t.ctypes.data))
    return c, t


def bgtq_get_layout(state, layer, kv_head):
    ng = ctypes.c_int32()
    w = np.zeros(4, dtype=np.int32)
    s = np.zeros(4, dtype=np.int32)
    perm = np.zeros(HEAD_DIM, dtype=np.int32)
    _check(lib().bgtq_get_layout(state, layer, kv_head, ctypes.byref(ng), w.ctypes.data, s.ctypes.data, perm.ctypes.data))
    return ng.value, w, s, perm


def bgtq_get_rotation(state, layer, kv_head, kind, group=0):
    buf = np.zeros(HEAD_DIM * HEAD_DIM, dtype=np.float32)
    d = ctypes.c_int32()
    _check(lib().bgtq_get_rotation(state, layer, kv_head, kind, group, buf.ctypes.data, ctypes.byref(d)))
    return buf[: d.value * d.value].reshape(d.value, d.value).copy()


def bgtq_cache_offsets(state):
    out = np.zeros(4, dtype=np.uint64)
    _check(lib().bgtq_cache_offsets(state, out.ctypes.data))
    return [int(x) for x in out]


def bgtq_encode_append(state, layer, layer_count, d_k, d_v, d_start, d_count, batch, n, stream=None):
    _check(lib().bgtq_encode_append(state, layer, layer_count, _ptr(d_k), _ptr(d_v), _ptr(d_start), _ptr(d_count),
                                    batch, n, _stream(stream)))


def bgtq_encode_append_rope(state, layer, layer_count, d_k, d_v, d_start, d_count, batch, n, rope_base,
                            stream=None):
    _check(lib().bgtq_encode_append_rope(state, layer, layer_count, _ptr(d_k), _ptr(d_v), _ptr(d_start),
                                         _ptr(d_count), batch, n, float(rope_base), _stream(stream)))


def bgtq_rotate_query(state, layer, layer_count, d_q, batch, d_qrot, stream=None):
    _check(lib().bgtq_rotate_query(state, layer, layer_count, _ptr(d_q), batch, _ptr(d_qrot), _stream(stream)))


def bgtq_decode_attn(state, layer, layer_count, d_q, d_seq_lens, batch, d_out, stream=None):
    _check(lib().bgtq_decode_attn(state, layer, layer_count, _ptr(d_q), _ptr(d_seq_lens), batch, _ptr(d_out),
                                  _stream(stream)))


def bgtq_decode_attn_buffered(state, layer, layer_count, d_q, d_seq_lens, d_pos_lo, batch, d_buf_k, d_buf_v,
                              d_buf_count, n_buf, d_out, stream=None):
    _check(lib().bgtq_decode_attn_buffered(state, layer, layer_count, _ptr(d_q), _ptr(d_seq_lens), _ptr(d_pos_lo),
                                           batch, _ptr(d_buf_k), _ptr(d_buf_v), _ptr(d_buf_count), n_buf,
                                           _ptr(d_out), _stream(stream)))


def bgtq_logit_mae(state, layer, layer_count, seq, w0, m, d_q, d_k, d_mae, stream=None):
    _check(lib().bgtq_logit_mae(state, layer, layer_count, seq, w0, m, _ptr(d_q), _ptr(d_k), _ptr(d_mae),
                                _stream(stream)))


def bgtq_set_block_table(state, d_block_table):
    _check(lib().bgtq_set_block_table(state, _ptr(d_block_table)))


def bgtq_decode_step(state, layer, layer_count, d_k, d_v, d_start, d_count, n, d_q, d_seq_lens, batch, d_out,
                     stream=None):
    _check(lib().bgtq_decode_step(state, layer, layer_count, _ptr(d_k), _ptr(d_v), _ptr(d_start), _ptr(d_count), n,
                                  _ptr(d_q), _ptr(d_seq_lens), batch, _ptr(d_out), _stream(stream)))


def bgtq_decode_step_buffered(state, layer, layer_count, d_k, d_v, d_start, d_count, n, d_q, d_seq_lens, d_pos_lo,
                              batch, d_buf_k, d_buf_v, d_buf_count, n_buf, d_out, stream=None):
    _check(lib().bgtq_decode_step_buffered(state, layer, layer_count, _ptr(d_k), _ptr(d_v), _ptr(d_start),
                                           _ptr(d_count), n, _ptr(d_q), _ptr(d_seq_lens), _ptr(d_pos_lo), batch,
                                           _ptr(d_buf_k), _ptr(d_buf_v), _ptr(d_buf_count), n_buf, _ptr(d_out),
                                           _stream(stream)))


def bgtq_decode_split(state, layer, layer_count, d_qrot, d_seq_lens, batch, stream=None):
    _check(lib().bgtq_decode_split(state, layer, layer_count, _ptr(d_qrot), _ptr(d_seq_lens), batch, _stream(stream)))


def bgtq_decode_combine(state, layer, layer_count, d_seq_lens, batch, d_out, stream=None):
    _check(lib().bgtq_decode_combine(state, layer, layer_count, _ptr(d_seq_lens), batch, _ptr(d_out), _stream(stream)))


def bgtq_decode_attn_static_scratch(state, layer, layer_count, d_q, d_seq_lens, batch, d_out, stream=None):
    """bgtq_decode_attn with the split-K scratch in the library's static device
    array (for callers that cannot allocate device memory)."""
    _check(lib().bgtq_decode_attn_static_scratch(state, layer, layer_count, _ptr(d_q), _ptr(d_seq_lens), batch,
                                                 _ptr(d_out), _stream(stream)))


def bgtq_set_split_tokens(state, tokens):
    _check(lib().bgtq_set_split_tokens(state, tokens))


def bgtq_set_decode_path(state, fused):
    _check(lib().bgtq_set_decode_path(state, int(fused)))


def bgtq_get_decode_path(state):
    """(fused, ctas): fused 1 when the decode calls run as one fused launch (0: query
    rotation, split pass and combine); ctas the CTAs one wave of that kernel holds."""
    out, ctas = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().bgtq_get_decode_path(state, ctypes.byref(out), ctypes.byref(ctas)))
    return out.value, ctas.value


def bgtq_get_device_error(state, stream=None):
    f = ctypes.c_int32()
    _check(lib().bgtq_get_device_error(state, _stream(stream), ctypes.byref(f)))
    return f.value


def bgtq_error_string(status):
    return lib().bgtq_error_string(status).decode()


class PackedKVCache:
    """One library state over torch-owned device buffers."""

    def __init__(self, cfg, device="cuda"):
        import torch
        self.cfg = cfg
        self.device = torch.device(device)
        self.cache_bytes, self.workspace_bytes = bgtq_required_bytes(cfg)
        self.cache = torch.zeros(self.cache_bytes, dtype=torch.uint8, device=self.device)
        self.workspace = torch.zeros(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.state = bgtq_create(cfg, self.cache, self.cache_bytes, self.workspace, self.workspace_bytes)
        self.offsets = bgtq_cache_offsets(self.state)

    def close(self):
        if getattr(self, "state", None):
            bgtq_destroy(self.state)
            self.state = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- views of the cache arrays (no copies) --
    def _tiles(self):
        """Leading dims of the cache arrays: (L, B, Hkv, T) contiguous, (L, Hkv, pages) paged."""
        c = self.cfg
        if c.page_pool_tiles > 0:
            return (c.n_layers, c.n_kv_heads, c.page_pool_tiles)
        return (c.n_layers, c.max_batch, c.n_kv_heads, (c.capacity_tokens + TILE - 1) // TILE)

    def k_tiles(self):
        t = self._tiles()
        n = int(np.prod(t)) * 1024 * self.cfg.k_avg_bits
        return self.cache[self.offsets[0]:self.offsets[0] + n].view(*t, 1024 * self.cfg.k_avg_bits)

    def k_norms(self):
        import torch
        t = self._tiles()
        n = int(np.prod(t)) * TILE * 8
        return self.cache[self.offsets[1]:self.offsets[1] + n].view(torch.float16).view(*t[:-1], t[-1] * TILE, 4)

    def v_tiles(self):
        t = self._tiles()
        n = int(np.prod(t)) * 1024 * self.cfg.v_avg_bits
        return self.cache[self.offsets[2]:self.offsets[2] + n].view(*t, 1024 * self.cfg.v_avg_bits)

    def v_norms(self):
        import torch
        t = self._tiles()
        n = int(np.prod(t)) * TILE * 2
        return self.cache[self.offsets[3]:self.offsets[3] + n].view(torch.float16).view(*t[:-1], t[-1] * TILE)

    # -- calls --
    # Every tensor is checked against the layout its call reads (see _expect)
    # before its pointer is passed on; counts and ranges are checked by the
    # library itself.
    def _q_like(self, t, name, layer_count, dtype):
        _expect(t, name, (layer_count, None, self.cfg.n_q_heads, HEAD_DIM), dtype, self.device)
        return t.shape[1]

    def _per_seq(self, t, name, batch):
        import torch
        _expect(t, name, (batch,), torch.int32, self.device)

    def _rows(self, k, v, start, count, layer_count, batch=None):
        """Checks appended rows k, v [layer_count, batch, n, Hkv, 128] (batch None: any) and
        start, count [batch]; returns (batch, n)."""
        import torch
        _expect(k, "k", (layer_count, batch, None, self.cfg.n_kv_heads, HEAD_DIM), torch.float16, self.device)
        _expect(v, "v", tuple(k.shape), torch.float16, self.device)
        self._per_seq(start, "start", k.shape[1])
        self._per_seq(count, "count", k.shape[1])
        return k.shape[1], k.shape[2]

    def allocate(self, calib_q, calib_k):
        """calib_q fp16 [n_layers, Nq, Hq, 128], calib_k fp16 [n_layers, Nk, Hkv, 128] on the device."""
        import torch
        c = self.cfg
        _expect(calib_q, "calib_q", (c.n_layers, None, c.n_q_heads, HEAD_DIM), torch.float16, self.device)
        _expect(calib_k, "calib_k", (c.n_layers, None, c.n_kv_heads, HEAD_DIM), torch.float16, self.device)
        bgtq_allocate(self.state, calib_q, calib_q.shape[1], calib_k, calib_k.shape[1])

    def set_allocation(self, widths):
        """int8 widths [n_layers, n_kv_heads, 64] (host)."""
        w = np.asarray(widths)
        if w.shape != (self.cfg.n_layers, self.cfg.n_kv_heads, N_BLOCKS):
            raise BgtqError(ERR_INVALID_ARG, f"widths: shape {w.shape}, expected "
                                             f"{(self.cfg.n_layers, self.cfg.n_kv_heads, N_BLOCKS)}")
        bgtq_set_allocation(self.state, w)

    def get_allocation(self):
        return bgtq_get_allocation(self.state, self.cfg.n_layers, self.cfg.n_kv_heads)

    def encode_append(self, layer, k, v, start, count, layer_count=1, rope_base=None):
        """k, v fp16 [layer_count, batch, n, Hkv, 128]; start, count int32 [batch] on the device.
        rope_base given: k is taken before RoPE and turned inside the encode
        (bgtq_encode_append_rope)."""
        batch, n = self._rows(k, v, start, count, layer_count)
        if rope_base is None:
            bgtq_encode_append(self.state, layer, layer_count, k, v, start, count, batch, n)
        else:
            bgtq_encode_append_rope(self.state, layer, layer_count, k, v, start, count, batch, n, rope_base)

    def rotate_query(self, layer, q, out, layer_count=1):
        """q fp16 and out fp32 [layer_count, batch, Hq, 128] on the device."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float32, self.device)
        bgtq_rotate_query(self.state, layer, layer_count, q, batch, out)

    def decode_attn(self, layer, q, seq_lens, out, layer_count=1):
        """q, out fp16 [layer_count, batch, Hq, 128]; seq_lens int32 [batch] on the device."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float16, self.device)
        self._per_seq(seq_lens, "seq_lens", batch)
        bgtq_decode_attn(self.state, layer, layer_count, q, seq_lens, batch, out)

    def decode_attn_static_scratch(self, layer, q, seq_lens, out, layer_count=1):
        """decode_attn with its scratch in the library's static device array
        (bgtq_decode_attn_static_scratch): same tensors, checked the same way."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float16, self.device)
        self._per_seq(seq_lens, "seq_lens", batch)
        bgtq_decode_attn_static_scratch(self.state, layer, layer_count, q, seq_lens, batch, out)

    def decode_step(self, layer, k, v, start, count, q, seq_lens, out, layer_count=1):
        """encode_append(k, v, start, count) then decode_attn(q, seq_lens, out), in one call (the appends
        and the query rotation share a launch when k holds at most 16 rows per sequence); k = None
        appends nothing."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float16, self.device)
        self._per_seq(seq_lens, "seq_lens", batch)
        n = 0 if k is None else self._rows(k, v, start, count, layer_count, batch)[1]
        bgtq_decode_step(self.state, layer, layer_count, k, v, start, count, n, q, seq_lens, batch, out)

    def _buffer(self, seq_lens, pos_lo, buf_k, buf_v, buf_count, layer_count, batch):
        import torch
        self._per_seq(seq_lens, "seq_lens", batch)
        self._per_seq(pos_lo, "pos_lo", batch)
        _expect(buf_k, "buf_k", (layer_count, batch, None, self.cfg.n_kv_heads, HEAD_DIM), torch.float16,
                self.device)
        _expect(buf_v, "buf_v", tuple(buf_k.shape), torch.float16, self.device)
        self._per_seq(buf_count, "buf_count", batch)
        return buf_k.shape[2]

    def decode_attn_buffered(self, layer, q, seq_lens, pos_lo, buf_k, buf_v, buf_count, out, layer_count=1):
        """Attention over the packed positions [pos_lo, seq_lens) and the first
        buf_count fp16 buffered rows (buf_k, buf_v fp16 [layer_count, batch,
        n_buf, Hkv, 128])."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float16, self.device)
        n_buf = self._buffer(seq_lens, pos_lo, buf_k, buf_v, buf_count, layer_count, batch)
        bgtq_decode_attn_buffered(self.state, layer, layer_count, q, seq_lens, pos_lo, batch, buf_k, buf_v,
                                  buf_count, n_buf, out)

    def logit_mae(self, layer, seq, w0, q, k, out, layer_count=1):
        """Per-head logit MAE of the packed keys at positions [w0, w0 + m) of
        sequence seq: q fp16 [layer_count, m, Hq, 128], k (exact keys) fp16
        [layer_count, m, Hkv, 128], out float64 [layer_count, Hq]."""
        import torch
        m = self._q_like(q, "q", layer_count, torch.float16)
        _expect(k, "k", (layer_count, m, self.cfg.n_kv_heads, HEAD_DIM), torch.float16, self.device)
        _expect(out, "out", (layer_count, self.cfg.n_q_heads), torch.float64, self.device)
        bgtq_logit_mae(self.state, layer, layer_count, seq, w0, m, q, k, out)

    def decode_step_buffered(self, layer, k, v, start, count, q, seq_lens, pos_lo, buf_k, buf_v, buf_count, out,
                             layer_count=1):
        """encode_append(k, v, start, count) then decode_attn_buffered(...), in one call; k = None
        appends nothing."""
        import torch
        batch = self._q_like(q, "q", layer_count, torch.float16)
        _expect(out, "out", tuple(q.shape), torch.float16, self.device)
        n_buf = self._buffer(seq_lens, pos_lo, buf_k, buf_v, buf_count, layer_count, batch)
        n = 0 if k is None else self._rows(k, v, start, count, layer_count, batch)[1]
        bgtq_decode_step_buffered(self.state, layer, layer_count, k, v, start, count, n, q, seq_lens, pos_lo,
                                  batch, buf_k, buf_v, buf_count, n_buf, out)

    def decode_split(self, layer, qrot, seq_lens, layer_count=1):
        """The split-K stage alone from rotated queries (fp32 [layer_count, batch, Hq, 128])."""
        import torch
        batch = self._q_like(qrot, "qrot", layer_count, torch.float32)
        self._per_seq(seq_lens, "seq_lens", batch)
        bgtq_decode_split(self.state, layer, layer_count, qrot, seq_lens, batch)

    def decode_combine(self, layer, seq_lens, out, layer_count=1):
        """The combine stage alone: out fp16 [layer_count, batch, Hq, 128]."""
        import torch
        batch = self._q_like(out, "out", layer_count, torch.float16)
        self._per_seq(seq_lens, "seq_lens", batch)
        bgtq_decode_combine(self.state, layer, layer_count, seq_lens, batch, out)

    def set_block_table(self, table):
        """Paged cache: int32 [max_batch, ceil(capacity / 64)] page ids on the
        device (kept referenced here; its contents are read at kernel time).
        A contiguous cache rejects any table."""
        import torch
        c = self.cfg
        if c.page_pool_tiles > 0 and table is not None:
            _expect(table, "table", (c.max_batch, (c.capacity_tokens + TILE - 1) // TILE), torch.int32, self.device)
        bgtq_set_block_table(self.state, table)
        self._block_table = table

    def test_drop_tile_copies(self, tile):
        """Test hook: the split pass skips the copies of cache tile `tile` (-1: off)."""
        _check(lib().bgtq_test_drop_tile_copies(self.state, tile))

    def set_split_tokens(self, tokens):
        bgtq_set_split_tokens(self.state, tokens)

    def set_decode_path(self, fused):
        """1: decode_attn / decode_step run as one fused launch where the GPU can; 0: three launches."""
        bgtq_set_decode_path(self.state, fused)

    def decode_path_fused(self):
        """True when decode_attn / decode_step run as one fused launch (bgtq_get_decode_path)."""
        return bgtq_get_decode_path(self.state)[0] == 1

    def decode_wave_ctas(self):
        """CTAs one wave of the decode kernel holds (the automatic split plan's budget)."""
        return bgtq_get_decode_path(self.state)[1]

    def device_error(self):
        return bgtq_get_device_error(self.state)
