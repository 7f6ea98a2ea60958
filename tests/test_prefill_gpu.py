"""Chunked prefill through the four decode calls, against the causal whole-sequence forward.

A chunk of T new tokens of one sequence is run as T batch entries that share
the sequence's page-table row: the append writes the chunk's T rows at
positions p0..p0+T-1, and entry t attends with seq_len = p0 + t + 1, so each
token sees the rows before it and itself and none after ("解耦 RoPE（MLA 下）"
§七 ``forward_naive``: token t attends to tokens 0..t).  Two chunks per
sequence; the second one attends over the first one's cached rows.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import synth
from mla_latent_kv_45_b200.layer import DecodeLayer
from mla_testlib import (assert_bf16_close, assert_fp32_close, dev, dev_weights, host,
                         lib_dims, oracle_dims)

pytestmark = pytest.mark.gpu


def _prefill(wl, chunks):
    W = synth.make_weights(wl)
    T = sum(chunks)
    hs = synth.make_hidden(wl, n=T)                      # one sequence, T tokens
    dims = lib_dims(wl)
    wl_cache = dataclasses.replace(wl, batch=1, new_tokens=T)
    pc = synth.make_paged_cache(wl_cache, np.zeros(1, dtype=np.int64), fill=False)
    pool = dev_pool(pc)
    outs = []
    p0 = 0
    for n in chunks:
        # n entries sharing the sequence's page-table row
        bt = torch.from_numpy(np.repeat(pc.block_table[:1], n, axis=0).astype(np.int32)).cuda()
        lens = torch.arange(p0 + 1, p0 + n + 1, dtype=torch.int32, device="cuda")
        cache = L.PagedCache(pool, bt, lens)
        layer = DecodeLayer(dims, dev_weights(W, wl), n)
        pos = torch.arange(p0, p0 + n, dtype=torch.int32, device="cuda")
        out = layer.step(cache, dev(hs[p0:p0 + n], wl), pos)
        assert layer.device_error() == 0
        outs.append(host(out).copy())
        p0 += n
    ref = oracle.forward_naive(hs, W, oracle_dims(wl))
    return np.concatenate(outs), ref


def dev_pool(pc):
    if pc.pool.dtype == np.uint16:
        return torch.from_numpy(pc.pool.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(pc.pool).cuda()


def test_tiny_fp32_chunked_prefill_matches_naive_forward():
    out, ref = _prefill(synth.TINY, [20, 13])
    assert_fp32_close(out, ref, "prefill u")


def test_bf16_chunked_prefill_matches_naive_forward():
    wl = synth.reduced(synth.V2_STEP128, "prefill", 41, 1, 0, 0)
    out, ref = _prefill(wl, [70, 45])   # ragged chunks over 64-row pages
    assert_bf16_close(out, ref, "prefill u")
