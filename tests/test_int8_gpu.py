"""The int8 latent cache (MLA_CACHE_INT8) on the GPU, against the fp64 oracle.

A row holds c as int8 codes times a power-of-two scale and k_R in bf16
("DeepSeek-V3多头潜在注意力(MLA)架构", 多头潜在注意力与KV缓存优化: the KV cache
stored at INT8 / INT4 precision).  Since q * 2^e is exact in bf16, attention
over an int8 pool must give bit-identical z and lse to attention over a bf16
pool holding the dequantised rows, and both must match the oracle on those
rows.  The append quantises with the oracle's rule (tightest power-of-two
scale, codes rounded half to even); the kernel forms c in fp32, so a code may
differ by one where c / s falls within fp32 error of a half-integer.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth
from mla_latent_kv_45_b200.layer import DecodeLayer

from mla_testlib import (LSE_ATOL, LSE_RTOL, assert_bf16_close, bf16_ulp, dev, dev_weights, host,
                         lib_dims, oracle_dims)

pytestmark = pytest.mark.gpu

V2 = synth.reduced(synth.V2_BATCH64, "int8", 81, 7, 0, 0, new_tokens=0)
LENS = np.array([1, 63, 64, 65, 700, 129, 3000])


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    L.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def i8_dims(wl):
    return dataclasses.replace(lib_dims(wl), cache_format=L.MLA_CACHE_INT8)


def dequant_rows(pc, b, n):
    codes, exps, k_r = pc.fields(b, n)
    return np.concatenate([oracle.dequantize_int8_pow2(codes, exps), k_r], axis=1)


def cache_of(pool_np, bt, lens):
    return L.PagedCache(torch.from_numpy(pool_np).cuda(),
                        torch.from_numpy(np.ascontiguousarray(bt, dtype=np.int32)).cuda(),
                        torch.from_numpy(np.asarray(lens, dtype=np.int32)).cuda())


def run(dims, cache, q, batch, splits):
    n = L.mla_workspace_size(dims, batch, 64, 0, splits)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    z = torch.empty(batch, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(batch, 128, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, q, z, lse, splits, ws)
    assert L.mla_get_device_error(ws) == 0
    return z, lse


@pytest.mark.parametrize("splits", [0, 3, 16])
def test_int8_attention_matches_oracle_and_bf16_pool(splits):
    pc = synth.make_paged_cache_int8(V2, LENS, spare_pages=1)
    q = synth.make_q_lat(V2)
    qd = dev(q, V2)
    z8, l8 = run(i8_dims(V2), cache_of(pc.pool, pc.block_table, LENS), qd, len(LENS), splits)
    # the same rows, dequantised, in a bf16 pool with the same page table
    bf = np.zeros(pc.pool.shape[:2] + (576,), dtype=np.uint16)
    for b, Lb in enumerate(LENS):
        idx = np.arange(Lb)
        bf[pc.block_table[b][idx // 64], idx % 64] = synth.bf16_bits(dequant_rows(pc, b, Lb))
    bf_cache = cache_of(bf.view(np.int16), pc.block_table, LENS)
    bf_cache.pool = bf_cache.pool.view(torch.bfloat16)
    zb, lb = run(lib_dims(V2), bf_cache, qd, len(LENS), splits)
    assert torch.equal(z8, zb) and torch.equal(l8, lb)
    od = oracle_dims(V2)
    zh, lh = host(z8), host(l8)
    for b, Lb in enumerate(LENS):
        zr, lr = oracle.attend_latent(q[b], dequant_rows(pc, b, Lb), od)
        assert_bf16_close(zh[b], zr, f"seq {b} len {Lb}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


def test_int8_append_quantises_like_the_oracle():
    wl = synth.reduced(synth.V2_BATCH64, "int8_app", 82, 4, 0, 0)
    prior = np.array([0, 63, 64, 1000])
    W = synth.make_weights(wl, seeded_gamma=True)
    pc = synth.make_paged_cache_int8(wl, prior, spare_pages=1)
    h = synth.make_hidden(wl)
    dims = i8_dims(wl)
    cache = cache_of(pc.pool, pc.block_table, prior + 1)
    before = cache.pool.clone()
    n = L.mla_workspace_size(dims, wl.batch, 5120, 0, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    Wd = dev_weights(W, wl)
    L.mla_cache_append(dims, cache, dev(h, wl), Wd["W_DKV"], Wd["W_KR"], Wd["gamma"],
                       torch.tensor(prior.astype(np.int32), device="cuda"), ws)
    assert L.mla_get_device_error(ws) == 0
    ref = oracle.latent_row(h, W["W_DKV"], W["W_KR"], W["gamma"], prior, oracle_dims(wl))
    q_ref, e_ref = oracle.quantize_int8_pow2(ref[:, :512])
    got = synth.Int8PagedCache(cache.pool.cpu().numpy(), pc.block_table, prior + 1, 64)
    changed = (cache.pool != before).any(-1).cpu().numpy()
    slots = set()
    exact = 0
    for b in range(wl.batch):
        p = prior[b]
        slots.add((pc.block_table[b][p // 64], p % 64))
        codes, exps, k_r = got.fields(b, p + 1)
        raw = got.raw_rows(b, p + 1)[-1]
        assert exps[-1] == e_ref[b], b
        assert np.all(np.abs(codes[-1] - q_ref[b]) <= 1), b
        exact += int((codes[-1] == q_ref[b]).sum())
        kr = ref[b, 512:]
        assert np.all(np.abs(k_r[-1] - oracle.bf16_round(kr)) <= bf16_ulp(kr) * 1.0001)
        assert np.all(raw[644:] == 0)
    assert {tuple(x) for x in np.argwhere(changed)} <= slots
    assert exact / (wl.batch * 512) > 0.99


def test_int8_full_step():
    """Append (quantised) + absorb + attention over the int8 cache + un-absorb."""
    wl = synth.reduced(synth.V2_STEP128, "int8_step", 83, 3, 0, 0)
    prior = np.array([10, 500, 1500])
    W = synth.make_weights(wl)
    pc = synth.make_paged_cache_int8(wl, prior)
    h = synth.make_hidden(wl)
    cache = cache_of(pc.pool, pc.block_table, prior + 1)
    layer = DecodeLayer(i8_dims(wl), dev_weights(W, wl), wl.batch)
    out = layer.step(cache, dev(h, wl), torch.tensor(prior.astype(np.int32), device="cuda"))
    assert layer.device_error() == 0
    od = oracle_dims(wl)
    # the oracle's step over the dequantised prior rows, with the new row
    # quantised by the oracle's rule
    new = oracle.latent_row(h, W["W_DKV"], W["W_KR"], W["gamma"], prior, od)
    qn, en = oracle.quantize_int8_pow2(new[:, :512])
    new_deq = np.concatenate([oracle.dequantize_int8_pow2(qn, en), new[:, 512:]], axis=1)
    ref_q = oracle.absorb_q(h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], prior, od)
    zs = []
    for b in range(wl.batch):
        rows = np.concatenate([dequant_rows(pc, b, prior[b]), new_deq[b:b + 1]])
        zs.append(oracle.attend_latent(ref_q[b], rows, od)[0])
    _, u = oracle.unabsorb(np.stack(zs), W["W_UV"], W["W_O"], od)
    assert_bf16_close(host(layer.z), np.stack(zs), "z")
    assert_bf16_close(host(out), u, "u")
