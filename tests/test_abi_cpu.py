"""C-ABI checks that need no GPU: the library loads, exports every symbol
``include/mla.h`` declares, and rejects bad arguments on the host before any
launch (fake, never-dereferenced addresses are enough for that)."""

import ctypes
import os
import re

import pytest

from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return L.lib()


def header_symbols():
    src = open(os.path.join(ROOT, "include", "mla.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", src)))


def test_header_symbols_exported(lib):
    syms = header_symbols()
    assert "mla_decode_attn" in syms and len(syms) >= 8
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(L.EXPORTS)


def test_split_kv_host_checks(lib):
    d = V2.c()
    c = _cache()
    p = lib.mla_decode_attn_partial
    assert p(ctypes.byref(d), ctypes.byref(c), 2, A, A, A, None, 0, A, 1 << 30, None) == 1
    assert p(ctypes.byref(d), ctypes.byref(c), 2, A, A + 8, A, A, 0, A, 1 << 30, None) == 3
    assert p(ctypes.byref(d), ctypes.byref(c), 2, A, A, A, A, 0, A, 100, None) == 4
    m = lib.mla_merge_partials
    assert m(ctypes.byref(d), 2, 0, A, A, A, A, None, None) == 1       # no parts
    assert m(ctypes.byref(d), 2, 3, A + 4, A, A, A, None, None) == 3   # O misaligned
    assert m(ctypes.byref(d), 2, 3, A, A, A, None, None, None) == 1    # null z


def test_status_strings(lib):
    for code in range(8):
        assert L.status_string(code)
    assert "aligned" in L.status_string(3)


V2 = L.Dims(128, 512, 64, 128, 128, 64, L.MLA_BF16)
TINY = L.Dims(4, 16, 8, 8, 8, 16, L.MLA_FP32)
A = 0x10000  # a fake 16-byte-aligned device address (never dereferenced)


def _cache(pool=A, bt=A, lens=A, num_pages=8, maxp=4):
    return L._Cache(pool, num_pages, bt, maxp, lens)


def attn(lib, dims, cache, batch=2, q=A, z=A, lse=None, splits=0, ws=A, wsb=1 << 30):
    d = dims.c()
    return lib.mla_decode_attn(ctypes.byref(d), ctypes.byref(cache), batch, q, z, lse, splits, ws,
                               wsb, None)


def test_workspace_size(lib):
    n = L.mla_workspace_size(V2, 64, 5120, 1536, 0)
    assert n > 64 * 128 * 512 * 4
    assert L.mla_workspace_size(V2, 64, 5120, 1536, 8) < n
    assert L.mla_workspace_size(L.Dims(128, 513, 64, 128, 128, 64), 4, 5120, 0, 0) == 0
    assert L.mla_workspace_size(TINY, 2, 64, 0, 0) > 0
    assert L.mla_workspace_size(L.Dims(4, 18, 8, 8, 8, 16, L.MLA_FP32), 2, 64, 0, 0) == 0


def test_decode_attn_host_checks(lib):
    bad = L.Dims(128, 513, 64, 128, 128, 64)
    assert attn(lib, bad, _cache()) == 2                     # unsupported bf16 shape
    assert attn(lib, L.Dims(128, 512, 63, 128, 128, 64), _cache()) == 1   # odd d_rope
    assert attn(lib, V2, _cache(), q=None) == 1              # null q_lat
    assert attn(lib, V2, _cache(pool=None)) == 1             # null pool
    assert attn(lib, V2, _cache(num_pages=0)) == 1
    assert attn(lib, V2, _cache(), batch=0) == 1
    assert attn(lib, V2, _cache(), q=A + 8) == 3             # misaligned
    assert attn(lib, V2, _cache(pool=A + 2)) == 3
    assert attn(lib, V2, _cache(), splits=-1) == 1
    assert attn(lib, V2, _cache(), wsb=100) == 4             # workspace too small
    assert attn(lib, V2, _cache(), ws=None) == 1
    t = L.Dims(4, 16, 8, 8, 8, 16, 7)                        # bad dtype enum
    assert attn(lib, t, _cache()) == 1
    i8 = L.Dims(128, 512, 64, 128, 128, 64, L.MLA_BF16, cache_format=L.MLA_CACHE_INT8)
    assert attn(lib, i8, _cache(), wsb=100) == 4             # int8 rows accepted (bf16 sizes)
    assert attn(lib, L.Dims(4, 16, 8, 8, 8, 16, L.MLA_FP32, cache_format=L.MLA_CACHE_INT8),
                _cache()) == 2                               # int8 rows need the bf16 path
    assert attn(lib, L.Dims(128, 512, 64, 128, 128, 64, cache_format=5), _cache()) == 1


def test_append_absorb_unabsorb_host_checks(lib):
    d = V2.c()
    c = _cache()
    f = lib.mla_cache_append
    assert f(ctypes.byref(d), ctypes.byref(c), 2, 5120, A, A, A, A, None, A, 1 << 30, None) == 1
    assert f(ctypes.byref(d), ctypes.byref(c), 2, 5000, A, A, A, A, A, A, 1 << 30, None) == 2
    assert f(ctypes.byref(d), ctypes.byref(c), 2, 5120, A + 4, A, A, A, A, A, 1 << 30, None) == 3
    assert f(ctypes.byref(d), ctypes.byref(c), 2, 5120, A, A, A, A, A, A, 10, None) == 4
    g = lib.mla_absorb_q
    assert g(ctypes.byref(d), 2, 5120, A, None, 1536, A, A, A, A, A, A, 1 << 30, None) == 1
    assert g(ctypes.byref(d), 2, 5120, A, A, 1500, A, A, A, A, A, A, 1 << 30, None) == 2
    assert g(ctypes.byref(d), 2, 5120, A, A, 1536, A, A, A, A, A + 2, A, 1 << 30, None) == 3
    u = lib.mla_unabsorb_out
    assert u(ctypes.byref(d), 2, A, A, A, 5000, A, A, 1 << 30, None) == 2
    assert u(ctypes.byref(d), 2, None, A, A, 5120, A, A, 1 << 30, None) == 1
    assert u(ctypes.byref(d), 2, A, A, A, 5120, A + 1, A, 1 << 30, None) == 3
    assert lib.mla_get_device_error(None, None) == 1
    assert lib.mla_workspace_init(None, 0, None) == 1
    assert lib.mla_workspace_init(A, 16, None) == 4


def test_library_does_not_route_through_oracle():
    """The product package never imports the oracle (test infrastructure)."""
    pkg = os.path.join(ROOT, "mla_latent_kv_45_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn), encoding="utf-8").read()
            assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), fn
