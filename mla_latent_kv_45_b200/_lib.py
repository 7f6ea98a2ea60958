"""ctypes binding of ``libmla_b200.so`` (declared in ``include/mla.h``).

Argument marshalling only: every function here forwards torch tensors' device
pointers and sizes to the C ABI call of the same name and raises ``MlaError``
on a non-OK status.  There is no fallback: if the library is missing the
import fails.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_b200.so")

MLA_BF16, MLA_FP32 = 0, 1
MLA_ROPE_INTERLEAVED, MLA_ROPE_HALF = 0, 1
MLA_CACHE_NATIVE, MLA_CACHE_INT8 = 0, 1
MLA_INT8_ROW_BYTES = 656

STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
          3: "MLA_ERR_ALIGNMENT", 4: "MLA_ERR_WORKSPACE", 5: "MLA_ERR_CUDA",
          6: "MLA_ERR_DEVICE_RANGE", 7: "MLA_ERR_TIMEOUT"}

EXPORTS = ("mla_workspace_size", "mla_workspace_init", "mla_cache_append", "mla_absorb_q",
           "mla_decode_attn", "mla_decode_attn_partial", "mla_merge_partials",
           "mla_decode_attn_noalloc", "mla_unabsorb_out",
           "mla_noalloc_get_device_error", "mla_get_device_error", "mla_debug_absorb_timeout",
           "mla_status_string")


class MlaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({status_string(status)})")


class _Dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int), ("d_c", ctypes.c_int), ("d_rope", ctypes.c_int),
                ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int), ("page_size", ctypes.c_int),
                ("dtype", ctypes.c_int), ("rope_layout", ctypes.c_int),
                ("rope_base", ctypes.c_double), ("rms_eps", ctypes.c_double),
                ("softmax_scale", ctypes.c_double), ("cache_format", ctypes.c_int)]


class _Cache(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("num_pages", ctypes.c_int),
                ("block_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int),
                ("seq_lens", ctypes.c_void_p)]


@dataclasses.dataclass
class Dims:
    """Mirror of ``mla_dims``."""
    n_heads: int
    d_c: int
    d_rope: int
    d_nope: int
    d_v: int
    page_size: int
    dtype: int = MLA_BF16
    rope_layout: int = MLA_ROPE_INTERLEAVED
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    softmax_scale: float = 0.0
    cache_format: int = MLA_CACHE_NATIVE

    def c(self) -> _Dims:
        return _Dims(*dataclasses.astuple(self))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == MLA_BF16 else torch.float32


@dataclasses.dataclass
class PagedCache:
    """Mirror of ``mla_paged_cache`` holding the torch tensors.

    pool ``[num_pages, page_size, d_c + d_rope]``, block_table
    ``[batch, max_pages_per_seq]`` int32, seq_lens ``[batch]`` int32.
    """
    pool: torch.Tensor
    block_table: torch.Tensor
    seq_lens: torch.Tensor

    def c(self) -> _Cache:
        return _Cache(self.pool.data_ptr(), self.pool.shape[0], self.block_table.data_ptr(),
                      self.block_table.shape[1], self.seq_lens.data_ptr())


_lib = None


def lib() -> ctypes.CDLL:
    """Loads the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m mla_latent_kv_45_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        pd, pc = ctypes.POINTER(_Dims), ctypes.POINTER(_Cache)
        L.mla_workspace_size.argtypes = [pd, i, i, i, i]
        L.mla_workspace_size.restype = sz
        L.mla_workspace_init.argtypes = [vp, sz, vp]
        L.mla_cache_append.argtypes = [pd, pc, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
        L.mla_absorb_q.argtypes = [pd, i, i, vp, vp, i, vp, vp, vp, vp, vp, vp, sz, vp]
        L.mla_decode_attn.argtypes = [pd, pc, i, vp, vp, vp, i, vp, sz, vp]
        L.mla_decode_attn_partial.argtypes = [pd, pc, i, vp, vp, vp, vp, i, vp, sz, vp]
        L.mla_merge_partials.argtypes = [pd, i, i, vp, vp, vp, vp, vp, vp]
        L.mla_decode_attn_noalloc.argtypes = [pd, pc, i, vp, vp, vp, i, vp]
        L.mla_unabsorb_out.argtypes = [pd, i, vp, vp, vp, i, vp, vp, sz, vp]
        L.mla_get_device_error.argtypes = [vp, vp]
        L.mla_noalloc_get_device_error.argtypes = [vp]
        L.mla_debug_absorb_timeout.argtypes = [i, ctypes.c_uint]
        L.mla_status_string.argtypes = [i]
        L.mla_status_string.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("mla_workspace_size", "mla_status_string"):
                getattr(L, name).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mla_status_string(status).decode()


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ok(fn: str, st: int):
    if st != 0:
        raise MlaError(fn, st)


def mla_workspace_size(dims: Dims, batch: int, d_model: int, d_q: int, num_splits: int = 0) -> int:
    d = dims.c()
    return int(lib().mla_workspace_size(ctypes.byref(d), batch, d_model, d_q, num_splits))


def mla_workspace_init(ws: torch.Tensor, stream=None):
    _ok("mla_workspace_init", lib().mla_workspace_init(_p(ws), ws.numel() * ws.element_size(),
                                                       _stream(stream)))


def mla_cache_append(dims: Dims, cache: PagedCache, h, W_DKV, W_KR, gamma, positions,
                     ws: torch.Tensor, stream=None):
    d, c = dims.c(), cache.c()
    _ok("mla_cache_append", lib().mla_cache_append(
        ctypes.byref(d), ctypes.byref(c), h.shape[0], h.shape[1], _p(h), _p(W_DKV), _p(W_KR),
        _p(gamma), _p(positions), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def mla_absorb_q(dims: Dims, x, W_DQ, W_UQ, W_QR, W_UK, positions, q_lat, ws: torch.Tensor,
                 stream=None):
    d = dims.c()
    d_q = W_DQ.shape[0] if W_DQ is not None else x.shape[1]
    _ok("mla_absorb_q", lib().mla_absorb_q(
        ctypes.byref(d), x.shape[0], x.shape[1], _p(x), _p(W_DQ), d_q, _p(W_UQ), _p(W_QR),
        _p(W_UK), _p(positions), _p(q_lat), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def mla_decode_attn(dims: Dims, cache: PagedCache, q_lat, z, lse=None, num_splits: int = 0,
                    ws: torch.Tensor = None, stream=None):
    d, c = dims.c(), cache.c()
    _ok("mla_decode_attn", lib().mla_decode_attn(
        ctypes.byref(d), ctypes.byref(c), q_lat.shape[0], _p(q_lat), _p(z), _p(lse), num_splits,
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def mla_decode_attn_partial(dims: Dims, cache: PagedCache, q_lat, O, m, l, num_splits: int = 0,
                            ws: torch.Tensor = None, stream=None):
    """Unnormalised partial softmax (O, m, l) over the rows this cache holds."""
    d, c = dims.c(), cache.c()
    _ok("mla_decode_attn_partial", lib().mla_decode_attn_partial(
        ctypes.byref(d), ctypes.byref(c), q_lat.shape[0], _p(q_lat), _p(O), _p(m), _p(l),
        num_splits, _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def mla_merge_partials(dims: Dims, O, m, l, z, lse=None, stream=None):
    """z (and lse) from partials stacked as O [n, B, H, d_c], m and l [n, B, H]."""
    d = dims.c()
    _ok("mla_merge_partials", lib().mla_merge_partials(
        ctypes.byref(d), O.shape[1], O.shape[0], _p(O), _p(m), _p(l), _p(z), _p(lse),
        _stream(stream)))


def mla_decode_attn_noalloc(dims: Dims, cache: PagedCache, q_lat, z, lse=None,
                            num_splits: int = 0, stream=None):
    """Decode attention with the library's fixed internal scratch (no workspace)."""
    d, c = dims.c(), cache.c()
    _ok("mla_decode_attn_noalloc", lib().mla_decode_attn_noalloc(
        ctypes.byref(d), ctypes.byref(c), q_lat.shape[0], _p(q_lat), _p(z), _p(lse), num_splits,
        _stream(stream)))


def mla_unabsorb_out(dims: Dims, z, W_UV, W_O, out, ws: torch.Tensor, stream=None):
    d = dims.c()
    d_model = W_O.shape[0] if W_O is not None else 0
    _ok("mla_unabsorb_out", lib().mla_unabsorb_out(
        ctypes.byref(d), z.shape[0], _p(z), _p(W_UV), _p(W_O), d_model, _p(out), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def mla_noalloc_get_device_error(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status of the last
    allocation-free decode-attention call on the current device."""
    return int(lib().mla_noalloc_get_device_error(_stream(stream)))


def mla_debug_absorb_timeout(enable: bool, wait_limit_us: int = 0):
    """Test hook: make the absorption kernel's q_C hand-off wait run out (see mla.h)."""
    _ok("mla_debug_absorb_timeout", lib().mla_debug_absorb_timeout(int(enable), wait_limit_us))


def mla_get_device_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns the device status code (0 = OK) and clears it."""
    return int(lib().mla_get_device_error(_p(ws), _stream(stream)))
