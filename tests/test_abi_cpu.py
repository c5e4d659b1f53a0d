"""CPU checks of the C-ABI library: it loads and exports every declared symbol."""
import os
import re

import pytest

from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import build as pkg_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bgtq.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bgtq_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    pkg_build.build()
    return bgtq.lib()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = header_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(bgtq.declared_symbols()) == names


def _header_prototypes():
    """{name: (return type, [parameter declarations])} from include/bgtq.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for ret, name, args in re.findall(r"([A-Za-z_][\w\s\*]*?)\b(bgtq_[a-z_]+)\s*\(([^)]*)\)\s*;", text):
        params = [a.strip() for a in args.split(",") if a.strip() and a.strip() != "void"]
        out[name] = (" ".join(ret.split()), params)
    return out


def _ctype_of(decl):
    """The ctypes type a C parameter declaration must be bound with (None: any
    pointer type, c_void_p or a typed ctypes pointer)."""
    import ctypes
    if "*" in decl:
        return None
    base = decl.rsplit(" ", 1)[0]
    return {"int32_t": ctypes.c_int32, "size_t": ctypes.c_size_t, "double": ctypes.c_double}[base]


def test_binding_signatures_match_the_header(lib):
    """Every ctypes signature has the header's parameter count and, parameter
    by parameter, the same kind (pointer, int32, size_t) and return type: a
    mismatch would shift every later argument of the call."""
    import ctypes
    protos = _header_prototypes()
    assert sorted(protos) == header_functions()
    for name, (ret, params) in protos.items():
        res, args = bgtq._SIGS[name]
        assert len(args) == len(params), (name, len(args), len(params))
        for decl, bound in zip(params, args):
            want = _ctype_of(decl)
            if want is None:
                assert bound is ctypes.c_void_p or issubclass(bound, ctypes._Pointer), (name, decl)
            else:
                assert bound is want, (name, decl, bound)
        if ret == "void":
            assert res is None, name
        elif ret == "int":
            assert res is ctypes.c_int, name
        else:
            assert ret.startswith("const char") and res is ctypes.c_char_p, (name, ret)


def test_error_strings(lib):
    assert bgtq.bgtq_error_string(0) == "ok"
    assert bgtq.bgtq_error_string(-1) == "invalid argument"
    assert bgtq.bgtq_error_string(-999) == "unknown status"


def test_required_bytes_is_host_only_and_validates(lib):
    cfg = bgtq.Config(n_layers=36, n_kv_heads=2, n_q_heads=16, max_batch=1, capacity_tokens=131072)
    cache, ws = bgtq.bgtq_required_bytes(cfg)
    toks = 36 * 2 * 131072
    assert cache >= toks * (48 + 8 + 48 + 2)
    assert cache < toks * (48 + 8 + 48 + 2) + 4 * 256
    assert cache % 256 == 0 and ws % 256 == 0
    bad = [dict(head_dim=64), dict(n_q_heads=15), dict(k_avg_bits=5), dict(b_min=4, b_max=3),
           dict(k_avg_bits=1, b_min=2), dict(rope_pairing=2), dict(capacity_tokens=0), dict(max_splits=2000),
           dict(page_pool_tiles=-1), dict(n_layers=65536),
           # sizes past 2^56 bytes (they would overflow the buffer plan's arithmetic)
           dict(n_layers=65535, max_batch=2 ** 31 - 1, capacity_tokens=2 ** 30),
           dict(n_layers=65535, n_kv_heads=2 ** 20, n_q_heads=2 ** 20, max_batch=2 ** 20)]
    for change in bad:
        c = bgtq.Config(**{**cfg.__dict__, **change})
        with pytest.raises(bgtq.BgtqError) as e:
            bgtq.bgtq_required_bytes(c)
        assert e.value.status == -1
    # the largest layer count is accepted and sized exactly like a smaller one, per layer
    one, _ = bgtq.bgtq_required_bytes(bgtq.Config(n_layers=1, n_kv_heads=1, n_q_heads=1, max_batch=1,
                                                  capacity_tokens=64))
    most, _ = bgtq.bgtq_required_bytes(bgtq.Config(n_layers=65535, n_kv_heads=1, n_q_heads=1, max_batch=1,
                                                   capacity_tokens=64))
    assert 65535 * (one - 1024) <= most <= 65535 * one


def test_paged_cache_is_sized_by_its_pool(lib):
    """A paged cache holds page_pool_tiles 64-position pages per (layer, KV
    head), whatever max_batch and capacity are; the workspace is unchanged."""
    base = dict(n_layers=28, n_kv_heads=4, n_q_heads=28, max_batch=16, capacity_tokens=32768, k_avg_bits=3,
                v_avg_bits=2)
    cont, ws = bgtq.bgtq_required_bytes(bgtq.Config(**base))
    pool = 6000   # about 16 sequences of U[16K, 32K] tokens
    paged, ws_p = bgtq.bgtq_required_bytes(bgtq.Config(**base, page_pool_tiles=pool))
    per_page = 64 * (48 + 8 + 32 + 2)
    assert 28 * 4 * pool * per_page <= paged < 28 * 4 * pool * per_page + 4 * 256
    assert cont >= 28 * 4 * 16 * 512 * per_page
    assert ws_p == ws


def test_library_fails_loudly_when_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(bgtq, "_lib", None)
    monkeypatch.setattr(bgtq, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError):
        bgtq.lib()
