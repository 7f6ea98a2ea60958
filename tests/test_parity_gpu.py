"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

fp32 validation mode: relative error <= 1e-4 (max|g-r| / max|r|).
bf16: max-abs <= 2e-2 and mean-rel <= 5e-3 on attention and projection outputs;
cache writes: placement bit-exact, values within one bf16 ulp of the
correctly rounded oracle value.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth
from mla_latent_kv_45_b200.layer import DecodeLayer

from mla_testlib import (LSE_ATOL, LSE_RTOL, assert_bf16_close, assert_fp32_close, bf16_ulp, dev,
                         dev_cache, dev_weights, host, lib_dims, metrics, oracle_dims)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    L.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def new_ws(dims, batch, d_model=64, d_q=0, splits=0):
    n = L.mla_workspace_size(dims, batch, d_model, d_q, splits)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    return ws


def ipos(a):
    return torch.tensor(np.asarray(a, dtype=np.int32), device="cuda")


# ---------------------------------------------------------------------------
# fp32 validation mode, tiny sizes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layout", [0, 1])
def test_tiny_fp32_full_step(layout):
    wl = dataclasses.replace(synth.TINY, rope_layout=layout)
    W = synth.make_weights(wl, seeded_gamma=True)
    prior = synth.make_prior_lengths(wl)
    pc = synth.make_paged_cache(wl, prior, spare_pages=3)
    h = synth.make_hidden(wl)
    dims, od = lib_dims(wl), oracle_dims(wl)
    cache = dev_cache(pc, prior + 1)
    before = cache.pool.clone()
    layer = DecodeLayer(dims, dev_weights(W, wl), wl.batch)
    out = layer.step(cache, dev(h, wl), ipos(prior))
    assert layer.device_error() == 0
    ref = oracle.decode_step(h, [pc.rows_f32(b, prior[b]) for b in range(wl.batch)], W, od)
    changed = (cache.pool != before).any(-1).cpu().numpy()
    expect = np.zeros_like(changed)
    for b in range(wl.batch):
        p = prior[b]
        page, slot = pc.block_table[b][p // wl.page_size], p % wl.page_size
        expect[page, slot] = True
        assert_fp32_close(host(cache.pool[page, slot]), ref["row"][b], "row", tol=1e-5)
    assert np.array_equal(changed, expect & changed) and changed.sum() <= wl.batch
    assert_fp32_close(host(layer.q_lat), ref["q_lat"], "q_lat")
    assert_fp32_close(host(layer.z), ref["z"], "z")
    np.testing.assert_allclose(host(layer.lse), ref["lse"], rtol=1e-5, atol=1e-5)
    assert_fp32_close(host(out), ref["u"], "u")


def test_tiny_fp32_decode_loop_matches_naive_forward():
    """33 decode steps from an empty cache equal the causal whole-sequence forward
    (the pages' naive == absorbed check, run through the library)."""
    wl = synth.TINY
    W = synth.make_weights(wl)
    T = wl.prior_max + 1
    hs = synth.make_hidden(wl, n=wl.batch * T).reshape(wl.batch, T, wl.d_model)
    dims, od = lib_dims(wl), oracle_dims(wl)
    prior = np.zeros(wl.batch, dtype=np.int64)
    pc = synth.make_paged_cache(dataclasses.replace(wl, new_tokens=T), prior, fill=False)
    lens = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    cache = dev_cache(pc, np.zeros(wl.batch))
    cache.seq_lens = lens
    layer = DecodeLayer(dims, dev_weights(W, wl), wl.batch)
    outs = []
    for t in range(T):
        lens.fill_(t + 1)
        outs.append(host(layer.step(cache, dev(hs[:, t], wl), ipos([t] * wl.batch))).copy())
    assert layer.device_error() == 0
    for b in range(wl.batch):
        ref = oracle.forward_naive(hs[b], W, od)
        assert_fp32_close(np.stack([o[b] for o in outs]), ref, f"seq {b}")


# ---------------------------------------------------------------------------
# bf16, DeepSeek-V2 head / latent sizes
# ---------------------------------------------------------------------------

def test_bf16_decode_loop_matches_naive_forward():
    """Multi-step decode at the DeepSeek-V2 sizes: 24 steps from an empty cache,
    each appending its row through the library and attending over the rows the
    library appended before, against the oracle's causal whole-sequence forward
    (K and V rebuilt, fp64)."""
    wl = synth.reduced(synth.V2_BATCH64, "v2_loop", 27, 2, 0, 0)
    W = synth.make_weights(wl)
    T = 24
    hs = synth.make_hidden(wl, n=wl.batch * T).reshape(wl.batch, T, wl.d_model)
    dims, od = lib_dims(wl), oracle_dims(wl)
    pc = synth.make_paged_cache(dataclasses.replace(wl, new_tokens=T), np.zeros(wl.batch, dtype=np.int64),
                                fill=False)
    lens = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    cache = dev_cache(pc, np.zeros(wl.batch))
    cache.seq_lens = lens
    layer = DecodeLayer(dims, dev_weights(W, wl), wl.batch)
    outs = []
    for t in range(T):
        lens.fill_(t + 1)
        outs.append(host(layer.step(cache, dev(hs[:, t], wl), ipos([t] * wl.batch))).copy())
    assert layer.device_error() == 0
    for b in range(wl.batch):
        ref = oracle.forward_naive(hs[b], W, od)
        assert_bf16_close(np.stack([o[b] for o in outs]), ref, f"seq {b}")


V2R = synth.reduced(synth.V2_BATCH64, "v2_ragged", 20, 6, 0, 0)
RAGGED = np.array([1, 63, 64, 65, 700, 129])


def run_attn(wl, pc, q, lens, splits=0):
    """mla_decode_attn on host inputs; returns (z, lse, device status)."""
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    ws = new_ws(dims, wl.batch, splits=splits)
    z = torch.empty(wl.batch, wl.n_heads, wl.d_c, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.batch, wl.n_heads, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, dev(q, wl), z, lse, splits, ws)
    return z, lse, L.mla_get_device_error(ws)


def attn_case(lens, splits=0, wl=V2R, shuffle=True):
    wl = dataclasses.replace(wl, batch=len(lens), new_tokens=0, shuffle_pages=shuffle)
    pc = synth.make_paged_cache(wl, np.asarray(lens), spare_pages=2)
    q = synth.make_q_lat(wl)
    z, lse, st = run_attn(wl, pc, q, lens, splits)
    return wl, pc, q, z, lse, st


@pytest.mark.parametrize("splits", [0, 1, 3, 16])
def test_bf16_attn_ragged(splits):
    wl, pc, q, z, lse, st = attn_case(RAGGED, splits)
    assert st == 0
    od = oracle_dims(wl)
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(RAGGED):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        assert_bf16_close(zh[b], zr, f"z seq {b} len {Lb}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


@pytest.mark.parametrize("splits", [0, 3, 16])
def test_bf16_attn_step_tails(splits):
    """1 to 9 pages with a one-row and a full last page: the attention takes pages
    four at a time (two per CTA of the pair), so this covers every shape of a
    piece's last step, whole and cut into partitions."""
    lens = np.array([64 * n + r for n in range(9) for r in (1, 64)])
    wl, pc, q, z, lse, st = attn_case(lens, splits)
    assert st == 0
    od = oracle_dims(wl)
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(lens):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        assert_bf16_close(zh[b], zr, f"z seq {b} len {Lb}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


@pytest.mark.parametrize("splits", [0, 5, 40])
def test_bf16_attn_cost_balanced_plan_edges(splits):
    """The plan charges each sequence a few virtual pages with no rows, so a
    partition's range may start or end inside those, hold no rows at all, or
    cut a sequence anywhere: many one- and two-page sequences around a few long
    ones, with few and with many partitions."""
    lens = np.array([1, 64, 65, 2, 3000, 1, 1, 128, 129, 7, 1, 700, 64, 1, 2, 5000, 1, 63, 1, 2])
    wl, pc, q, z, lse, st = attn_case(lens, splits)
    assert st == 0
    od = oracle_dims(wl)
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(lens):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        assert_bf16_close(zh[b], zr, f"z seq {b} len {Lb}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


def test_bf16_attn_split_and_page_order_invariance():
    lens = np.array([900, 5, 300, 2000])
    _, _, _, z1, l1, _ = attn_case(lens, 1)
    _, _, _, z8, l8, _ = attn_case(lens, 8)
    m = metrics(host(z8), host(z1))
    assert m["max_abs"] <= 1e-2 and m["mean_rel"] <= 2e-3, m
    # shuffled vs identity page order: the same rows give bit-identical results
    _, _, _, za, la, _ = attn_case(lens, 8, shuffle=True)
    _, _, _, zb, lb, _ = attn_case(lens, 8, shuffle=False)
    assert torch.equal(za, zb) and torch.equal(la, lb)


@pytest.mark.parametrize("layout", [0, 1])
def test_bf16_cache_append(layout):
    wl = dataclasses.replace(synth.reduced(synth.V2_BATCH64, "v2_app", 21, 4, 0, 0),
                             rope_layout=layout)
    prior = np.array([0, 63, 64, 1000])
    W = synth.make_weights(wl, seeded_gamma=True)
    pc = synth.make_paged_cache(wl, prior, spare_pages=1)
    h = synth.make_hidden(wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, prior + 1)
    before = cache.pool.clone()
    ws = new_ws(dims, wl.batch, 5120)
    Wd = dev_weights(W, wl)
    L.mla_cache_append(dims, cache, dev(h, wl), Wd["W_DKV"], Wd["W_KR"], Wd["gamma"], ipos(prior),
                       ws)
    assert L.mla_get_device_error(ws) == 0
    ref = oracle.latent_row(h, W["W_DKV"], W["W_KR"], W["gamma"], prior, oracle_dims(wl))
    changed = (cache.pool.view(torch.int16) != before.view(torch.int16)).any(-1).cpu().numpy()
    slots = set()
    exact = 0
    for b in range(wl.batch):
        p = prior[b]
        page, slot = pc.block_table[b][p // 64], p % 64
        slots.add((page, slot))
        g = host(cache.pool[page, slot])
        r = ref[b]
        rr = oracle.bf16_round(r)
        assert np.all(np.abs(g - rr) <= bf16_ulp(r) * 1.0001), b
        exact += int((g == rr).sum())
    assert {tuple(x) for x in np.argwhere(changed)} <= slots
    assert exact / (wl.batch * wl.row) > 0.9


@pytest.mark.parametrize("with_dq,layout", [(True, 0), (False, 0), (True, 1)])
def test_bf16_absorb_q(with_dq, layout):
    wl = dataclasses.replace(synth.reduced(synth.V2_BATCH64, "v2_abs", 22, 5, 0, 0),
                             rope_layout=layout, d_q=1536 if with_dq else 0)
    W = synth.make_weights(wl)
    h = synth.make_hidden(wl)
    pos = np.array([0, 1, 4095, 70000, 131071])
    dims = lib_dims(wl)
    ws = new_ws(dims, wl.batch, 5120, wl.d_q)
    Wd = dev_weights(W, wl)
    q = torch.empty(wl.batch, 128, 576, dtype=torch.bfloat16, device="cuda")
    L.mla_absorb_q(dims, dev(h, wl), Wd["W_DQ"], Wd["W_UQ"], Wd["W_QR"], Wd["W_UK"], ipos(pos), q,
                   ws)
    assert L.mla_get_device_error(ws) == 0
    ref = oracle.absorb_q(h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], pos, oracle_dims(wl))
    g = host(q)
    assert_bf16_close(g[..., :512], ref[..., :512], "q~")
    assert_bf16_close(g[..., 512:], ref[..., 512:], "q_R")


@pytest.mark.parametrize("with_o", [True, False])
def test_bf16_unabsorb(with_o):
    wl = synth.reduced(synth.V2_BATCH64, "v2_unabs", 23, 5, 0, 0)
    W = synth.make_weights(wl)
    zin = synth.make_z(wl)
    dims = lib_dims(wl)
    ws = new_ws(dims, wl.batch, 5120)
    Wd = dev_weights(W, wl)
    n_out = 5120 if with_o else 128 * 128
    out = torch.empty(wl.batch, n_out, dtype=torch.bfloat16, device="cuda")
    L.mla_unabsorb_out(dims, dev(zin, wl), Wd["W_UV"], Wd["W_O"] if with_o else None, out, ws)
    assert L.mla_get_device_error(ws) == 0
    o, u = oracle.unabsorb(zin, W["W_UV"], W["W_O"] if with_o else None, oracle_dims(wl))
    assert_bf16_close(host(out), u if with_o else o, "out")


def test_bf16_full_step_small_batch():
    wl = synth.reduced(synth.V2_STEP128, "v2_step_small", 24, 3, 0, 0)
    prior = np.array([10, 500, 1500])
    W = synth.make_weights(wl)
    pc = synth.make_paged_cache(wl, prior)
    h = synth.make_hidden(wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, prior + 1)
    layer = DecodeLayer(dims, dev_weights(W, wl), wl.batch)
    out = layer.step(cache, dev(h, wl), ipos(prior))
    assert layer.device_error() == 0
    ref = oracle.decode_step(h, [pc.rows_f32(b, prior[b]) for b in range(3)], W, oracle_dims(wl))
    assert_bf16_close(host(layer.z), ref["z"], "z")
    assert_bf16_close(host(out), ref["u"], "u")


# ---------------------------------------------------------------------------
# Edge cases: device-side range checks never write out of bounds
# ---------------------------------------------------------------------------

def test_bf16_empty_and_bad_sequences():
    lens = np.array([100, 0, 64, 130])
    wl = dataclasses.replace(V2R, batch=4, new_tokens=0)
    pc = synth.make_paged_cache(wl, np.maximum(lens, 1))
    bt = pc.block_table.copy()
    bt[3][1] = pc.num_pages + 7          # an out-of-range page entry
    q = synth.make_q_lat(wl)
    dims = lib_dims(wl)
    cache = dev_cache(dataclasses.replace(pc, block_table=bt), lens)
    ws = new_ws(dims, 4)
    z = torch.full((4, 128, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(4, 128, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, dev(q, wl), z, lse, 0, ws)
    assert L.mla_get_device_error(ws) == 6      # MLA_ERR_DEVICE_RANGE
    assert L.mla_get_device_error(ws) == 0      # reading clears the word
    zh, lh = host(z), host(lse)
    for b in (1, 3):
        assert np.all(zh[b] == 0) and np.all(np.isneginf(lh[b]))
    od = oracle_dims(wl)
    for b in (0, 2):
        zr, _ = oracle.attend_latent(q[b], pc.rows_f32(b, lens[b]), od)
        assert_bf16_close(zh[b], zr, f"seq {b}")


def test_append_out_of_range_position():
    wl = synth.reduced(synth.V2_BATCH64, "v2_app_bad", 25, 2, 0, 0)
    prior = np.array([10, 20])
    W = synth.make_weights(wl)
    pc = synth.make_paged_cache(wl, prior)
    dims = lib_dims(wl)
    cache = dev_cache(pc, prior + 1)
    before = cache.pool.clone()
    ws = new_ws(dims, 2, 5120)
    Wd = dev_weights(W, wl)
    cap = pc.block_table.shape[1] * 64
    L.mla_cache_append(dims, cache, dev(synth.make_hidden(wl), wl), Wd["W_DKV"], Wd["W_KR"],
                       Wd["gamma"], ipos([cap + 5, -1]), ws)
    assert L.mla_get_device_error(ws) == 6
    assert torch.equal(cache.pool.view(torch.int16), before.view(torch.int16))


# ---------------------------------------------------------------------------
# Full-size workloads
# ---------------------------------------------------------------------------

def test_bf16_attn_batch64_full():
    """batch 64, cached lengths U[1024, 8192] + the new row, shuffled 64-row pages."""
    wl = dataclasses.replace(synth.V2_BATCH64, new_tokens=0)
    lens = synth.make_prior_lengths(synth.V2_BATCH64) + 1
    wl_l = dataclasses.replace(wl, prior_min=0, prior_max=0)
    pc = synth.make_paged_cache(wl_l, lens)
    q = synth.make_q_lat(wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    ws = new_ws(dims, wl.batch)
    z = torch.empty(wl.batch, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.batch, 128, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, dev(q, wl), z, lse, 0, ws)
    assert L.mla_get_device_error(ws) == 0
    zh, lh = host(z), host(lse)
    od = oracle_dims(wl)
    for b in range(wl.batch):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, lens[b]), od)
        assert_bf16_close(zh[b], zr, f"seq {b}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


def test_bf16_attn_long_sampled():
    """batch 8 x 131072 rows (split-KV); sequences 0 and 7 checked against the oracle."""
    wl = synth.V2_LONG
    lens = np.full(wl.batch, 131072)
    pc = synth.make_paged_cache(dataclasses.replace(wl, prior_min=0, prior_max=0), lens)
    q = synth.make_q_lat(wl)
    dims = lib_dims(wl)
    cache = dev_cache(pc, lens)
    ws = new_ws(dims, wl.batch)
    z = torch.empty(wl.batch, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.batch, 128, dtype=torch.float32, device="cuda")
    L.mla_decode_attn(dims, cache, dev(q, wl), z, lse, 0, ws)
    assert L.mla_get_device_error(ws) == 0
    zh, lh = host(z), host(lse)
    od = oracle_dims(wl)
    for b in (0, 7):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, lens[b]), od)
        assert_bf16_close(zh[b], zr, f"seq {b}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


# ---------------------------------------------------------------------------
# Softmax paths of the attention kernel
# ---------------------------------------------------------------------------
#
# The kernel takes a piece of a sequence in steps of STEP_ROWS rows and keeps a
# running maximum in log2 units that moves only when a step's maximum exceeds it
# by more than RESCALE_LOG2; only then is the accumulated O rescaled.

STEP_ROWS = 256
RESCALE_LOG2 = 8.0
SOFTMAX_LENS = np.array([1, 63, 65, 256, 257, 700, 3000, 5000])


def _set_rows(pc, b, rows):
    idx = np.arange(len(rows))
    pc.pool[pc.block_table[b][idx // pc.page_size], idx % pc.page_size] = synth.bf16_bits(rows)


def _ramp_case():
    """k_R of row s grows from x1 to x32 along each sequence, c stays N(0, 1):
    the position score, and with it each head's running maximum, rises step
    after step by far more than 2^8, while z stays a mean of N(0, 1) rows."""
    lens = SOFTMAX_LENS
    wl = dataclasses.replace(V2R, batch=len(lens), new_tokens=0)
    pc = synth.make_paged_cache(wl, lens, spare_pages=2)
    for b, Lb in enumerate(lens):
        rows = pc.rows_f32(b, Lb).copy()
        rows[:, 512:] *= (1.0 + 31.0 * np.arange(Lb) / max(Lb - 1, 1))[:, None]
        _set_rows(pc, b, rows)
    return wl, pc, synth.make_q_lat(wl)


@pytest.mark.parametrize("splits", [0, 1, 3, 16])
def test_bf16_attn_rescale_path(splits):
    wl, pc, q, = _ramp_case()
    od = oracle_dims(wl)
    # the inputs do drive the rescale: for every head of the long sequences the
    # maximum over the whole sequence exceeds the first step's by more than 2^8
    # (in log2 units), so an unsplit piece must move its running max at least once
    for b in (6, 7):
        lg = (q[b].astype(np.float64) @ pc.rows_f32(b, SOFTMAX_LENS[b]).T) * od.scale / np.log(2)
        assert np.all(lg.max(1) - lg[:, :STEP_ROWS].max(1) > 4 * RESCALE_LOG2)
    z, lse, st = run_attn(wl, pc, q, SOFTMAX_LENS, splits)
    assert st == 0
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(SOFTMAX_LENS):
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        assert_bf16_close(zh[b], zr, f"z seq {b} len {Lb}")
        np.testing.assert_allclose(lh[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


@pytest.mark.parametrize("splits", [0, 3, 16])
def test_bf16_attn_one_dominant_row(splits):
    """Every head shares one q_R; a planted row with k_R = 10 q_R scores ~40 nats
    above the rest, so z is that row's latent c: exactly, after the bf16 store."""
    lens = SOFTMAX_LENS
    wl = dataclasses.replace(V2R, batch=len(lens), new_tokens=0)
    pc = synth.make_paged_cache(wl, lens, spare_pages=2)
    q = synth.make_q_lat(wl).copy()
    u = q[:, 0, 512:].copy()
    q[:, :, 512:] = u[:, None, :]
    # first row, last row, a page's middle, the first row of a later step, ...
    where = [0, 62, 64, 255, 256, 699, 1536, 4999]
    for b, (Lb, p) in enumerate(zip(lens, where)):
        assert p < Lb
        rows = pc.rows_f32(b, Lb).copy()
        rows[p, 512:] = synth.round_bf16(10.0 * u[b])
        _set_rows(pc, b, rows)
    z, lse, st = run_attn(wl, pc, q, lens, splits)
    assert st == 0
    zh = host(z)
    od = oracle_dims(wl)
    for b, (Lb, p) in enumerate(zip(lens, where)):
        rows = pc.rows_f32(b, Lb)
        assert np.array_equal(zh[b], np.broadcast_to(rows[p, :512], zh[b].shape)), b
        zr, lr = oracle.attend_latent(q[b], rows, od)
        assert_bf16_close(zh[b], zr, f"seq {b}")
        np.testing.assert_allclose(host(lse)[b], lr, atol=LSE_ATOL, rtol=LSE_RTOL)


@pytest.mark.parametrize("splits", [0, 3, 16])
def test_bf16_attn_equal_scores(splits):
    """q_lat = 0: every score is 0, so z is the plain mean of the sequence's c rows
    (any row past the end that leaked in would move it) and lse = ln L."""
    lens = SOFTMAX_LENS
    wl = dataclasses.replace(V2R, batch=len(lens), new_tokens=0)
    pc = synth.make_paged_cache(wl, lens, spare_pages=2)
    # fill the unused slots of the last pages with large values
    for b, Lb in enumerate(lens):
        for s in range(Lb, -(-Lb // 64) * 64):
            pc.pool[pc.block_table[b][s // 64], s % 64] = synth.bf16_bits(np.full(576, 1e4))
    q = np.zeros((len(lens), 128, 576), np.float32)
    z, lse, st = run_attn(wl, pc, q, lens, splits)
    assert st == 0
    zh, lh = host(z), host(lse)
    for b, Lb in enumerate(lens):
        mean = pc.rows_f32(b, Lb)[:, :512].astype(np.float64).mean(0)
        assert_bf16_close(zh[b], np.broadcast_to(mean, zh[b].shape), f"seq {b}")
        np.testing.assert_allclose(lh[b], np.log(Lb), rtol=1e-6, atol=1e-6)


# ---------------------------------------------------------------------------
# Whole decode steps at the full workload sizes (z and the layer output u)
# ---------------------------------------------------------------------------

def full_step(wl, prior, W, pc, h):
    cache = dev_cache(pc, prior + 1)
    layer = DecodeLayer(lib_dims(wl), dev_weights(W, wl), wl.batch)
    out = layer.step(cache, dev(h, wl), ipos(prior))
    assert layer.device_error() == 0
    # absorbed form of the oracle (pinned equal to the un-absorbed one)
    ref = oracle.decode_step(h, [pc.rows_f32(b, prior[b]) for b in range(wl.batch)], W,
                             oracle_dims(wl), unabsorbed=False)
    assert_bf16_close(host(layer.q_lat), ref["q_lat"], "q_lat")
    zh = host(layer.z)
    for b in range(wl.batch):
        assert_bf16_close(zh[b], ref["z"][b], f"z seq {b}")
    np.testing.assert_allclose(host(layer.lse), ref["lse"], atol=LSE_ATOL, rtol=LSE_RTOL)
    assert_bf16_close(host(out), ref["u"], "u")


def test_bf16_full_step_v2_single():
    """batch 1, 4096 cached rows + the new one, W_DQ .. W_O: the smallest grid."""
    wl = synth.V2_SINGLE
    prior = synth.make_prior_lengths(wl)
    full_step(wl, prior, synth.make_weights(wl), synth.make_paged_cache(wl, prior),
              synth.make_hidden(wl))


def test_bf16_full_step_v2_step128():
    """batch 128, 2048 cached rows + the new one each, the whole layer step."""
    wl = synth.V2_STEP128
    prior = synth.make_prior_lengths(wl)
    full_step(wl, prior, synth.make_weights(wl), synth.make_paged_cache(wl, prior),
              synth.make_hidden(wl))


def test_bf16_full_step_bench_inputs():
    """The decode step on exactly the inputs bench.py times (rank 0's shard of
    batch 64, cached rows U[1024, 8192] + 1, shuffled pages)."""
    import bench
    wl = bench.workload("v2_batch64", 0)
    prior = synth.make_prior_lengths(wl)
    full_step(wl, prior, synth.make_weights(wl), synth.make_paged_cache(wl, prior),
              synth.make_hidden(wl))


def test_captured_step_matches_eager_step():
    """DecodeLayer.capture: replaying the captured step over new inputs copied
    into its buffers gives bit-identical outputs to the eager step."""
    wl = synth.reduced(synth.V2_STEP128, "v2_graph", 26, 3, 0, 0)
    prior = np.array([100, 640, 1999])
    W = synth.make_weights(wl)
    pc = synth.make_paged_cache(wl, prior)
    dims = lib_dims(wl)
    cache = dev_cache(pc, prior + 1)
    layer = DecodeLayer(dims, dev_weights(W, wl), wl.batch)
    hd = dev(synth.make_hidden(wl), wl)
    pos = ipos(prior)
    graph = layer.capture(cache, hd, pos)
    h2 = dev(synth.make_hidden(wl, tid=30), wl)
    hd.copy_(h2)
    got = graph.replay().clone()
    assert layer.device_error() == 0
    want = layer.step(cache, h2, pos).clone()
    assert layer.device_error() == 0
    assert torch.equal(got, want)
