"""Seeded synthetic inputs for MLA decode: weights, hidden states, cache pools.

This module only draws random numbers (NumPy PCG64) and rounds them to the
storage dtype; it holds none of the method's arithmetic.  Tests, the bench and
the CPU oracle all take their inputs from here, so both sides see the same
bytes.  Seeds are ``1000 * workload_id + tensor_id``.

Workloads (DeepSeek-V2 attention sizes from "从零理解 MLA", 实际配置:
128 heads, d_nope 128, d_c 512, d_rope 64, q_lora 1536; d_model 5120):

* ``tiny``   fp32 validation: batch 2, 4 heads, d_model 64, d_c 16, d_nope 8,
             d_rope 8, d_v 8, no query compression, 32 cached rows + 1 new,
             16-token pages.
* ``v2_single``  bf16, batch 1, 4096 cached rows + 1 new.
* ``v2_batch64`` bf16, batch 64, cached rows ~ U[1024, 8192] + 1 new, 64-token
             pages in shuffled pool order.
* ``v2_long``    bf16, batch 8, 131072 rows per sequence (positions 0..131071,
             the query's own row included), attention only.
* ``v2_step128`` bf16, batch 128, 2048 cached rows + 1 new, whole layer step.
* ``v2_batch64_int8``  ``v2_batch64`` over 656-byte int8 cache rows.
* ``v2_prefill256``    one sequence, 4096 cached rows, a 256-token chunk.

Distributions: weights N(0, 0.02^2), hidden states N(0, 1), RMSNorm gain 1
(optionally 1 + 0.1 N(0,1)), cached rows N(0, 1) (the scale of an
RMS-normalised latent; k_R likewise), absorbed queries N(0, 1).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


# ---------------------------------------------------------------------------
# bf16 storage helpers (input preparation only)
# ---------------------------------------------------------------------------

def bf16_bits(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (((b >> 16) & 1) + 0x7FFF).astype(np.uint32)
    return (b >> 16).astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x) -> np.ndarray:
    """float32 values rounded to the nearest bfloat16, returned as float32."""
    return bf16_to_f32(bf16_bits(x))


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


# ---------------------------------------------------------------------------
# Workload descriptions
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # seed base: 1000 * wid + tensor id
    batch: int
    n_heads: int
    d_model: int
    d_q: int                 # 0 = no query compression (queries from h)
    d_c: int
    d_nope: int
    d_rope: int
    d_v: int
    page_size: int
    dtype: str               # "bf16" | "fp32"
    prior_min: int           # cached rows before the step, per sequence
    prior_max: int
    new_tokens: int = 1      # new tokens per sequence (a chunk when > 1); 0 = attention only
    shuffle_pages: bool = True
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    rope_layout: int = 0     # 0 interleaved, 1 half-split
    cache: str = "native"    # "native": rows in `dtype`; "int8": 656-byte int8 rows

    @property
    def row(self) -> int:
        return self.d_c + self.d_rope


TINY = Workload("tiny", 0, 2, 4, 64, 0, 16, 8, 8, 8, 16, "fp32", 32, 32)
V2_SINGLE = Workload("v2_single", 1, 1, 128, 5120, 1536, 512, 128, 64, 128, 64, "bf16", 4096, 4096)
V2_BATCH64 = Workload("v2_batch64", 2, 64, 128, 5120, 1536, 512, 128, 64, 128, 64, "bf16", 1024, 8192)
V2_LONG = Workload("v2_long", 3, 8, 128, 5120, 1536, 512, 128, 64, 128, 64, "bf16", 131072, 131072,
                   new_tokens=0)
V2_STEP128 = Workload("v2_step128", 4, 128, 128, 5120, 1536, 512, 128, 64, 128, 64, "bf16", 2048, 2048)
# the batch-64 workload (same seeds) over an int8 latent cache
V2_BATCH64_INT8 = dataclasses.replace(V2_BATCH64, name="v2_batch64_int8", cache="int8")
# chunked prefill: one sequence, 4096 cached rows, a chunk of 256 new tokens
V2_PREFILL256 = Workload("v2_prefill256", 6, 1, 128, 5120, 1536, 512, 128, 64, 128, 64, "bf16",
                         4096, 4096, new_tokens=256)

WORKLOADS = {w.name: w for w in (TINY, V2_SINGLE, V2_BATCH64, V2_LONG, V2_STEP128,
                                 V2_BATCH64_INT8, V2_PREFILL256)}


def reduced(base: Workload, name: str, wid: int, batch: int, prior_min: int, prior_max: int,
            **kw) -> Workload:
    """A smaller workload with ``base``'s head and latent sizes."""
    return dataclasses.replace(base, name=name, wid=wid, batch=batch, prior_min=prior_min,
                               prior_max=prior_max, **kw)


# ---------------------------------------------------------------------------
# Draws
# ---------------------------------------------------------------------------

def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Values as stored on the device, returned as float32."""
    x = np.asarray(x, dtype=np.float32)
    return round_bf16(x) if dtype == "bf16" else x


def make_weights(wl: Workload, seeded_gamma: bool = False) -> dict:
    """Layer weights in ``[out, in]`` layout, as stored (float32 arrays)."""
    s = 1000 * wl.wid
    H = wl.n_heads
    d_in_q = wl.d_q if wl.d_q else wl.d_model

    def w(tid, shape):
        return _store(rng(s + tid).normal(0.0, 0.02, size=shape).astype(np.float32), wl.dtype)

    gamma = np.ones(wl.d_c, dtype=np.float32)
    if seeded_gamma:
        gamma = 1.0 + 0.1 * rng(s + 9).standard_normal(wl.d_c).astype(np.float32)
    return {
        "W_DKV": w(1, (wl.d_c, wl.d_model)),
        "W_KR": w(2, (wl.d_rope, wl.d_model)),
        "gamma": _store(gamma, wl.dtype),
        "W_DQ": w(3, (wl.d_q, wl.d_model)) if wl.d_q else None,
        "W_UQ": w(4, (H * wl.d_nope, d_in_q)),
        "W_QR": w(5, (H * wl.d_rope, d_in_q)),
        "W_UK": w(6, (H * wl.d_nope, wl.d_c)),
        "W_UV": w(7, (H * wl.d_v, wl.d_c)),
        "W_O": w(8, (wl.d_model, H * wl.d_v)),
    }


def make_hidden(wl: Workload, tid: int = 10, n: Optional[int] = None) -> np.ndarray:
    """Hidden states of the new tokens, ``[batch, d_model]`` (or ``[n, d_model]``)."""
    n = wl.batch if n is None else n
    return _store(rng(1000 * wl.wid + tid).standard_normal((n, wl.d_model), dtype=np.float32),
                  wl.dtype)


def make_prior_lengths(wl: Workload) -> np.ndarray:
    """Cached rows per sequence before the step, uniform in [prior_min, prior_max]."""
    if wl.prior_min == wl.prior_max:
        return np.full(wl.batch, wl.prior_min, dtype=np.int64)
    return rng(1000 * wl.wid + 11).integers(wl.prior_min, wl.prior_max + 1, size=wl.batch)


@dataclasses.dataclass
class PagedCache:
    """A paged latent pool and its page table, as host arrays.

    ``pool`` is ``[num_pages, page_size, d_c + d_rope]``: uint16 bf16 bits
    for bf16 workloads, float32 otherwise.  ``block_table[b][j]`` is the pool
    page holding rows ``j*page_size .. (j+1)*page_size-1`` of sequence b
    (-1 where the sequence has no page).  ``prior_lens[b]`` rows are filled;
    capacity covers ``prior_lens[b] + new_tokens`` rows.
    """
    pool: np.ndarray
    block_table: np.ndarray
    prior_lens: np.ndarray
    page_size: int

    @property
    def num_pages(self) -> int:
        return self.pool.shape[0]

    def rows_f32(self, b: int, length: int) -> np.ndarray:
        """Rows 0..length-1 of sequence b as float32 (exact)."""
        idx = np.arange(length)
        pages = self.block_table[b][idx // self.page_size]
        r = self.pool[pages, idx % self.page_size]
        return bf16_to_f32(r) if r.dtype == np.uint16 else r.astype(np.float32)


def make_paged_cache(wl: Workload, prior_lens: Optional[np.ndarray] = None,
                     spare_pages: int = 0, fill: bool = True) -> PagedCache:
    """Pool with ``prior_lens[b]`` seeded rows per sequence, pages shuffled.

    Rows are N(0, 1) (c and k_R alike).  Pages are assigned to sequences in
    order, then the pool order is permuted (seed ``1000*wid + 12``) when
    ``wl.shuffle_pages``.  Unfilled slots hold zeros.
    """
    if prior_lens is None:
        prior_lens = make_prior_lengths(wl)
    ps = wl.page_size
    cap = prior_lens + wl.new_tokens
    pages_per = (cap + ps - 1) // ps
    total = int(pages_per.sum()) + spare_pages
    max_pages = max(int(pages_per.max()), 1)
    perm = np.arange(total)
    if wl.shuffle_pages:
        perm = rng(1000 * wl.wid + 12).permutation(total)
    bt = np.full((wl.batch, max_pages), -1, dtype=np.int32)
    k = 0
    for b in range(wl.batch):
        for j in range(int(pages_per[b])):
            bt[b, j] = perm[k]
            k += 1
    store_dt = np.uint16 if wl.dtype == "bf16" else np.float32
    pool = np.zeros((total, ps, wl.row), dtype=store_dt)
    if fill:
        g = rng(1000 * wl.wid + 13)
        for b in range(wl.batch):
            L = int(prior_lens[b])
            if L == 0:
                continue
            vals = g.standard_normal((L, wl.row), dtype=np.float32)
            vals = bf16_bits(vals) if wl.dtype == "bf16" else vals
            idx = np.arange(L)
            pool[bt[b][idx // ps], idx % ps] = vals
    return PagedCache(pool, bt, np.asarray(prior_lens, dtype=np.int64), ps)


INT8_ROW_BYTES = 656


@dataclasses.dataclass
class Int8PagedCache:
    """A paged pool of 656-byte int8 rows and its page table, as host arrays.

    Row layout (the library's MLA_CACHE_INT8 format): bytes [0, 512) int8 codes
    of c, [512, 640) k_R as 64 bf16 values, [640, 644) the row's scale 2^e as
    an fp32 value, [644, 656) zero.  ``fields`` unpacks a sequence's rows
    exactly (codes, exponents, k_R); turning them into values is the method's
    arithmetic and left to the caller.
    """
    pool: np.ndarray          # [num_pages, page_size, 656] uint8
    block_table: np.ndarray
    prior_lens: np.ndarray
    page_size: int

    @property
    def num_pages(self) -> int:
        return self.pool.shape[0]

    def raw_rows(self, b: int, length: int) -> np.ndarray:
        idx = np.arange(length)
        return self.pool[self.block_table[b][idx // self.page_size], idx % self.page_size]

    def fields(self, b: int, length: int):
        r = self.raw_rows(b, length)
        codes = r[:, :512].view(np.int8).astype(np.int64)
        k_r = bf16_to_f32(np.ascontiguousarray(r[:, 512:640]).view(np.uint16))
        scale = np.ascontiguousarray(r[:, 640:644]).view(np.float32)[:, 0]
        exps = np.round(np.log2(scale)).astype(np.int64)
        return codes, exps, k_r


def make_paged_cache_int8(wl: Workload, prior_lens: Optional[np.ndarray] = None,
                          spare_pages: int = 0) -> Int8PagedCache:
    """Pool of int8 rows with the same page assignment as ``make_paged_cache``.

    Codes are round(32 N(0, 1)) clipped to [-127, 127], exponents uniform in
    [-9, -4] (so values q 2^e have roughly the spread of an RMS-normalised
    latent), k_R ~ N(0, 1) rounded to bf16.  Unfilled rows are zero bytes.
    """
    if prior_lens is None:
        prior_lens = make_prior_lengths(wl)
    ref = make_paged_cache(dataclasses.replace(wl, dtype="bf16"), prior_lens, spare_pages,
                           fill=False)
    pool = np.zeros(ref.pool.shape[:2] + (INT8_ROW_BYTES,), dtype=np.uint8)
    g = rng(1000 * wl.wid + 16)
    ps = wl.page_size
    for b in range(wl.batch):
        L = int(prior_lens[b])
        if L == 0:
            continue
        codes = np.clip(np.round(32.0 * g.standard_normal((L, 512))), -127, 127).astype(np.int8)
        exps = g.integers(-9, -3, size=L)
        k_r = bf16_bits(g.standard_normal((L, 64), dtype=np.float32))
        rows = np.zeros((L, INT8_ROW_BYTES), dtype=np.uint8)
        rows[:, :512] = codes.view(np.uint8)
        rows[:, 512:640] = k_r.view(np.uint8).reshape(L, 128)
        rows[:, 640:644] = np.exp2(exps).astype(np.float32).view(np.uint8).reshape(L, 4)
        idx = np.arange(L)
        pool[ref.block_table[b][idx // ps], idx % ps] = rows
    return Int8PagedCache(pool, ref.block_table, ref.prior_lens, ps)


def make_q_lat(wl: Workload, tid: int = 14) -> np.ndarray:
    """Absorbed queries ``[batch, n_heads, d_c + d_rope]`` ~ N(0, 1), as stored."""
    return _store(rng(1000 * wl.wid + tid).standard_normal((wl.batch, wl.n_heads, wl.row),
                                                             dtype=np.float32), wl.dtype)


def make_z(wl: Workload, tid: int = 15) -> np.ndarray:
    """Latent attention outputs ``[batch, n_heads, d_c]`` ~ N(0, 1/16), as stored."""
    return _store(0.25 * rng(1000 * wl.wid + tid).standard_normal((wl.batch, wl.n_heads, wl.d_c),
                                                                    dtype=np.float32), wl.dtype)
