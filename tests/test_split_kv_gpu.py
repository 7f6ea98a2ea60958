"""Cross-device split-KV kernels on one GPU: the partial softmax of a share of
each sequence's pages (mla_decode_attn_partial) and the merge of the shares
(mla_merge_partials), against the fp64 oracle.

The shares are made with ``split_kv.shard_pages`` as views of one pool (their
own page tables and row counts), so the kernels see exactly what each device
of a split would see; no kernel waits on another.  Each share is compared as
its normalised output O / l and its log-sum-exp m + log l (the kernel's m may
lag the true maximum by its lazy rescale, which changes O, m and l together but
not these two), and the merged z / lse as the full attention.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth
from mla_latent_kv_45_b200.split_kv import shard_pages

from mla_testlib import (LSE_ATOL, LSE_RTOL, assert_bf16_close, assert_fp32_close, dev, dev_cache,
                         host, lib_dims, oracle_dims)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    L.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.mark.parametrize("kind,world", [("bf16", 3), ("bf16", 8), ("fp32", 3)])
def test_partials_and_merge_match_oracle(kind, world):
    if kind == "bf16":
        lens = np.array([1, 63, 65, 700, 3000, 64 * 9])
        wl = synth.reduced(synth.V2_BATCH64, "split_kv_gpu", 71, len(lens), 0, 0, new_tokens=0)
        close, f32 = assert_bf16_close, False
    else:
        lens = np.array([1, 17, 70, 33])
        wl = dataclasses.replace(synth.TINY, name="split_kv_fp32", wid=72, batch=len(lens),
                                 new_tokens=0)
        close, f32 = assert_fp32_close, True
    pc = synth.make_paged_cache(wl, lens, spare_pages=1)
    q = synth.make_q_lat(wl)
    dims, od = lib_dims(wl), oracle_dims(wl)
    qd = dev(q, wl)
    B, H, d_c = wl.batch, wl.n_heads, wl.d_c
    shards = shard_pages(pc.block_table, lens, wl.page_size, world)
    n = L.mla_workspace_size(dims, B, 64, 0, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    gO = torch.empty(world, B, H, d_c, dtype=torch.float32, device="cuda")
    gm = torch.empty(world, B, H, dtype=torch.float32, device="cuda")
    gl = torch.empty(world, B, H, dtype=torch.float32, device="cuda")
    for r, (bt_r, lens_r) in enumerate(shards):
        cache = dev_cache(dataclasses.replace(pc, block_table=bt_r), lens_r)
        L.mla_decode_attn_partial(dims, cache, qd, gO[r], gm[r], gl[r], 0, ws)
        assert L.mla_get_device_error(ws) == 0      # empty shares are not errors
        O, m, l = host(gO[r]), host(gm[r]), host(gl[r])
        for b in range(B):
            k = int(lens_r[b])
            if k == 0:
                assert np.all(O[b] == 0) and np.all(np.isneginf(m[b])) and np.all(l[b] == 0)
                continue
            idx = np.arange(k)
            rows = pc.pool[bt_r[b][idx // wl.page_size], idx % wl.page_size]
            rows = synth.bf16_to_f32(rows) if rows.dtype == np.uint16 else rows
            Or, mr, lr = oracle.split_partial(q[b], rows, od)
            close(O[b] / l[b][:, None], Or / lr[:, None], f"share {r} seq {b}")
            np.testing.assert_allclose(m[b] + np.log(l[b]), mr + np.log(lr), atol=LSE_ATOL, rtol=LSE_RTOL)
    z = torch.empty(B, H, d_c, dtype=dims.torch_dtype, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    L.mla_merge_partials(dims, gO, gm, gl, z, lse)
    torch.cuda.synchronize()
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(lens):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        close(zh[b], zr, f"merged seq {b}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


def test_merge_of_only_empty_parts():
    wl = synth.reduced(synth.V2_BATCH64, "split_kv_empty", 73, 2, 0, 0, new_tokens=0)
    dims = lib_dims(wl)
    gO = torch.zeros(2, 2, 128, 512, dtype=torch.float32, device="cuda")
    gm = torch.full((2, 2, 128), float("-inf"), dtype=torch.float32, device="cuda")
    gl = torch.zeros(2, 2, 128, dtype=torch.float32, device="cuda")
    z = torch.full((2, 128, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 128, dtype=torch.float32, device="cuda")
    L.mla_merge_partials(dims, gO, gm, gl, z, lse)
    torch.cuda.synchronize()
    assert torch.all(z == 0) and torch.all(torch.isneginf(lse))
