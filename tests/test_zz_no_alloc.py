"""The allocation-free decode-attention entry point (mla_decode_attn_noalloc).

It serves callers that cannot allocate device memory: programs whose device
memory is fully owned by another allocator, and plugin interfaces that pass
only the operation's tensors and allow no allocation while it runs.  Its
scratch is a fixed array inside the library, so nothing here hands it a
workspace.  Each case calls it twice in a row through the C ABI and checks
both results against mla_decode_attn (which takes a caller workspace) on the
same inputs, within the tolerances the parity tests use.  This file is named to
be collected last; it needs no state from other tests.
"""

import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth

from mla_testlib import assert_bf16_close, assert_fp32_close, dev, dev_cache, host, lib_dims

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


@pytest.mark.parametrize("kind", ["bf16", "fp32"])
def test_noalloc_matches_workspace_entry_point(kind):
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
    q = dev(synth.make_q_lat(wl), wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    z_ref, lse_ref = _with_workspace(dims, cache, q, wl.batch)
    z = torch.empty_like(z_ref)
    lse = torch.empty_like(lse_ref)
    for call in range(2):
        z.fill_(3.0)
        lse.fill_(3.0)
        assert _noalloc_c_abi(dims, cache, q, z, lse) == 0
        torch.cuda.synchronize()
        close(host(z), host(z_ref), f"z, call {call}")
        np.testing.assert_allclose(host(lse), host(lse_ref), atol=2e-3, rtol=0)


def test_noalloc_rejects_oversize_request():
    lens = np.array([100, 200])
    wl = synth.reduced(synth.V2_BATCH64, "noalloc_big", 52, 2, 0, 0, new_tokens=0)
    pc = synth.make_paged_cache(wl, lens)
    q = dev(synth.make_q_lat(wl), wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    z = torch.full((2, 128, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 128, dtype=torch.float32, device="cuda")
    # 1000 partitions need ~500 MB of partials: beyond the fixed scratch
    assert _noalloc_c_abi(dims, cache, q, z, lse, splits=1000) == 4   # MLA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(z == 3.0)   # nothing was enqueued
