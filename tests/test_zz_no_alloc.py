"""The allocation-free decode-attention entry point (mla_decode_attn_noalloc).

It serves callers that cannot allocate device memory: programs whose device
memory is fully owned by another allocator, and plugin interfaces that pass
only the operation's tensors and allow no allocation while it runs.  Its
scratch is a fixed array inside the library, so nothing here hands it a
workspace.  Each case calls it twice in a row through the C ABI and checks
both results element by element against the fp64 oracle, and against
mla_decode_attn (which takes a caller workspace) on the same inputs, within the
tolerances the parity tests use.  Its device status is read back with
mla_noalloc_get_device_error.  This file is named to be collected last; it
needs no state from other tests.
"""

import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth

from mla_testlib import (LSE_ATOL, LSE_RTOL, assert_bf16_close, assert_fp32_close, dev, dev_cache,
                         host, lib_dims, oracle_dims)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    L.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _with_workspace(dims, cache, q, batch, splits=0):
    n = L.mla_workspace_size(dims, batch, 64, 0, splits)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    z = torch.empty(batch, dims.n_heads, dims.d_c, dtype=dims.torch_dtype, device="cuda")
    lse = torch.empty(batch, dims.n_heads, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, q, z, lse, splits, ws)
    assert L.mla_get_device_error(ws) == 0
    return z, lse


def _noalloc_c_abi(dims, cache, q, z, lse, splits=0):
    """Direct C-ABI call (no workspace argument exists)."""
    d, c = dims.c(), cache.c()
    return L.lib().mla_decode_attn_noalloc(ctypes.byref(d), ctypes.byref(c), q.shape[0],
                                           q.data_ptr(), z.data_ptr(), lse.data_ptr(), splits,
                                           torch.cuda.current_stream().cuda_stream)


def _noalloc_status():
    return L.lib().mla_noalloc_get_device_error(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("kind,splits", [("bf16", 0), ("bf16", 7), ("fp32", 0)])
def test_noalloc_matches_oracle_and_workspace_entry_point(kind, splits):
    if kind == "bf16":
        lens = np.array([1, 700, 5000, 64, 3000, 129])
        wl = synth.reduced(synth.V2_BATCH64, "noalloc_bf16", 50, len(lens), 0, 0, new_tokens=0)
        close = assert_bf16_close
    else:
        lens = np.array([33, 5, 70])
        wl = dataclasses.replace(synth.TINY, name="noalloc_fp32", wid=51, batch=len(lens),
                                 new_tokens=0)
        close = assert_fp32_close
    pc = synth.make_paged_cache(wl, lens, spare_pages=1)
    q_host = synth.make_q_lat(wl)
    q = dev(q_host, wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    od = oracle_dims(wl)
    ref = [oracle.attend_latent(q_host[b], pc.rows_f32(b, Lb), od) for b, Lb in enumerate(lens)]
    z_ws, lse_ws = _with_workspace(dims, cache, q, wl.batch, splits)
    z = torch.empty_like(z_ws)
    lse = torch.empty_like(lse_ws)
    for call in range(2):
        z.fill_(3.0)
        lse.fill_(3.0)
        assert _noalloc_c_abi(dims, cache, q, z, lse, splits) == 0
        assert _noalloc_status() == 0
        zh, lh = host(z), host(lse)
        for b in range(wl.batch):
            close(zh[b], ref[b][0], f"z seq {b}, call {call}")
            np.testing.assert_allclose(lh[b], ref[b][1], atol=LSE_ATOL, rtol=LSE_RTOL)
        close(zh, host(z_ws), f"z vs workspace entry point, call {call}")
        np.testing.assert_allclose(lh, host(lse_ws), atol=LSE_ATOL, rtol=LSE_RTOL)


def test_noalloc_int8_pool_matches_oracle_and_workspace_entry_point():
    """The same entry point over an int8-row pool (MLA_CACHE_INT8)."""
    lens = np.array([1, 700, 5000, 64, 129])
    wl = synth.reduced(synth.V2_BATCH64, "noalloc_int8", 54, len(lens), 0, 0, new_tokens=0)
    pc = synth.make_paged_cache_int8(wl, lens, spare_pages=1)
    q_host = synth.make_q_lat(wl)
    q = dev(q_host, wl)
    dims = dataclasses.replace(lib_dims(wl), cache_format=L.MLA_CACHE_INT8)
    cache = L.PagedCache(torch.from_numpy(pc.pool).cuda(),
                         torch.from_numpy(np.ascontiguousarray(pc.block_table, dtype=np.int32)).cuda(),
                         torch.from_numpy(lens.astype(np.int32)).cuda())
    od = oracle_dims(wl)
    ref = []
    for b, Lb in enumerate(lens):
        codes, exps, k_r = pc.fields(b, Lb)
        rows = np.concatenate([oracle.dequantize_int8_pow2(codes, exps), k_r], axis=1)
        ref.append(oracle.attend_latent(q_host[b], rows, od))
    z_ws, lse_ws = _with_workspace(dims, cache, q, wl.batch)
    z = torch.empty_like(z_ws)
    lse = torch.empty_like(lse_ws)
    assert _noalloc_c_abi(dims, cache, q, z, lse) == 0
    assert _noalloc_status() == 0
    zh, lh = host(z), host(lse)
    for b in range(wl.batch):
        assert_bf16_close(zh[b], ref[b][0], f"z seq {b}")
        np.testing.assert_allclose(lh[b], ref[b][1], atol=LSE_ATOL, rtol=LSE_RTOL)
    assert_bf16_close(zh, host(z_ws), "z vs workspace entry point")
    np.testing.assert_allclose(lh, host(lse_ws), atol=LSE_ATOL, rtol=LSE_RTOL)


def test_noalloc_reports_device_range_errors():
    lens = np.array([100, 130])
    wl = synth.reduced(synth.V2_BATCH64, "noalloc_bad", 53, 2, 0, 0, new_tokens=0)
    pc = synth.make_paged_cache(wl, lens)
    bt = pc.block_table.copy()
    bt[1][1] = pc.num_pages + 3            # an out-of-range page entry
    q_host = synth.make_q_lat(wl)
    dims = lib_dims(wl)
    cache = dev_cache(dataclasses.replace(pc, block_table=bt), lens)
    z = torch.full((2, 128, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 128, dtype=torch.float32, device="cuda")
    assert _noalloc_c_abi(dims, cache, dev(q_host, wl), z, lse) == 0
    assert _noalloc_status() == 6          # MLA_ERR_DEVICE_RANGE
    assert _noalloc_status() == 0          # reading clears it
    zh, lh = host(z), host(lse)
    assert np.all(zh[1] == 0) and np.all(np.isneginf(lh[1]))
    zr, _ = oracle.attend_latent(q_host[0], pc.rows_f32(0, lens[0]), oracle_dims(wl))
    assert_bf16_close(zh[0], zr, "seq 0")


def test_noalloc_rejects_oversize_request():
    lens = np.array([100, 200])
    wl = synth.reduced(synth.V2_BATCH64, "noalloc_big", 52, 2, 0, 0, new_tokens=0)
    pc = synth.make_paged_cache(wl, lens)
    q = dev(synth.make_q_lat(wl), wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    z = torch.full((2, 128, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 128, dtype=torch.float32, device="cuda")
    # 31 partitions need 16 MiB of partials alone: beyond the fixed scratch;
    # 1000 need ~500 MB
    for splits in (31, 1000):
        assert _noalloc_c_abi(dims, cache, q, z, lse, splits=splits) == 4   # MLA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(z == 3.0)   # nothing was enqueued
    assert _noalloc_c_abi(dims, cache, q, z, lse, splits=30) == 0
    assert _noalloc_status() == 0
    torch.cuda.synchronize()
