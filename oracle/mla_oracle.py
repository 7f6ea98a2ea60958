"""fp64 oracle: the plain definitions of every step of absorbed MLA decode.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Everything is float64
NumPy; inputs are the exact values the GPU sees (bf16 / fp32 numbers upcast
to float64).  Nothing is blocked, fused or reordered beyond what the
definitions state.

Notation follows the pages: ``h`` hidden state, ``c`` the 512-wide latent
(c_KV), ``k_R`` the shared pre-rotated RoPE key, ``c_Q`` the compressed query,
``q_C`` / ``q_R`` the content / position query, ``q_lat`` the absorbed query
``[W_UK,i^T q_C,i ; q_R,i]``, ``z`` the latent-space attention output,
``o`` the per-head value output and ``u`` the output projection.

Pins (tests/test_oracle_pins.py) -- every function below is pinned:

* ``rope``            hand example values (解耦 RoPE §4.3-4.5), relative-position
                      identity, shift invariance, layout permutation identity,
                      norm preservation, scalar brute force.
* ``rms_norm``        closed forms (RMS of the output, scale invariance), brute force.
* ``latent_row``      hand example k_R rows; brute force.
* ``queries``/``absorb_q``  hand example q_R; absorption identity against the
                      un-absorbed logits; brute force.
* ``attend_latent``   special cases (L = 1, equal scores, one dominant score,
                      plain MQA reduction), brute force, absorbed == un-absorbed.
* ``attend_unabsorbed``  hand example totals; naive-forward equivalence.
* ``split_partial`` / ``combine_splits``  one split is the identity; any split
                      equals the unsplit softmax.
* ``unabsorb``        absorption identity ``W_UV,i z_i == o_i``; brute force.
* ``forward_naive``   causal brute force; equals the step-by-step absorbed loop.
* ``gather_rows``     rows scattered one by one into a shuffled pool by the
                      layout's definition come back in logical order.
* ``quantize_int8_pow2`` / ``dequantize_int8_pow2``  closed forms (code range,
                      tightest scale, error <= s / 2), brute-force search of the
                      exponent, half-to-even ties, torch.round on c / s.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

ROPE_INTERLEAVED = 0
ROPE_HALF = 1

__all__ = [
    "ROPE_INTERLEAVED", "ROPE_HALF", "Dims", "bf16_round", "rope_inv_freq", "rope",
    "rms_norm", "latent_row", "queries", "absorb_q", "attend_latent",
    "attend_unabsorbed", "split_partial", "combine_splits", "unabsorb",
    "decode_step", "forward_naive", "absorbed_decode_loop", "gather_rows",
    "INT8_MAX", "quantize_int8_pow2", "dequantize_int8_pow2",
]


@dataclasses.dataclass(frozen=True)
class Dims:
    """Head / latent sizes of one MLA layer.

    DeepSeek-V2 values ("从零理解 MLA", 实际配置): n_heads 128, d_nope 128,
    d_c 512, d_rope 64, q_lora (d_c') 1536.  ``softmax_scale`` 0 means
    1/sqrt(d_nope + d_rope) ("解耦 RoPE（MLA 下）" §4.6 note; "从零理解 MLA",
    解耦 RoPE: the scale becomes sqrt(d_head + d_r)).
    """

    n_heads: int
    d_c: int
    d_rope: int
    d_nope: int
    d_v: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    softmax_scale: float = 0.0
    rope_layout: int = ROPE_INTERLEAVED

    @property
    def scale(self) -> float:
        if self.softmax_scale:
            return float(self.softmax_scale)
        return 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def row(self) -> int:
        """Values cached per token: d_c + d_rope (576 at DeepSeek-V2 sizes)."""
        return self.d_c + self.d_rope


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def bf16_round(x) -> np.ndarray:
    """Round-to-nearest-even of float64 values to the nearest bfloat16.

    Used only to state what a bf16 store of an exact result should hold
    (the comparison target of the cache-write test).  Two-step rounding
    through float32 can double-round, so the rounding is done directly on the
    float64 value: the bfloat16 grid at ``x`` has spacing
    2**(floor(log2|x|) - 7) in the normal range.
    """
    x = _f64(x)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    e = np.maximum(e, -126.0)  # subnormal spacing stays 2**-133
    ulp = np.exp2(e - 7.0)
    q = x[nz] / ulp
    out[nz] = np.round(q) * ulp  # np.round is round-half-to-even
    return out


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def rope_inv_freq(d_rope: int, base: float) -> np.ndarray:
    """theta_i = base ** (-2 i / d_rope), i = 0 .. d_rope/2 - 1.

    "解耦 RoPE（MLA 下）" §七 ``rope`` (theta = base ** (-i/d) over even i);
    "从零理解 MLA", 解耦 RoPE ``precompute_cos_sin`` (same frequencies).  With
    d_rope = 2 this is the hand example's theta = 1 (§四).
    """
    i = np.arange(d_rope // 2, dtype=np.float64)
    return float(base) ** (-2.0 * i / float(d_rope))


def rope(x, pos, base: float = 10000.0, layout: int = ROPE_INTERLEAVED) -> np.ndarray:
    """Rotate the last axis of ``x`` by position ``pos`` (angles in float64).

    A pair (x0, x1) at frequency theta_i turns by pos * theta_i:
    (x0 cos - x1 sin, x0 sin + x1 cos) -- "解耦 RoPE（MLA 下）" §四 (the
    2-D rotation rule) and §七 ``rope``.

    ``layout`` picks the pairing:
      ROPE_INTERLEAVED  pairs (0,1), (2,3), ... ("解耦 RoPE（MLA 下）" §七);
      ROPE_HALF         pairs (i, i + d/2)     ("从零理解 MLA", 解耦 RoPE
                        ``apply_rope``, the half-split pairing).
    ``pos`` broadcasts against ``x.shape[:-1]``.
    """
    x = _f64(x)
    d = x.shape[-1]
    if d % 2:
        raise ValueError("RoPE needs an even width")
    ang = _f64(pos)[..., None] * rope_inv_freq(d, base)
    cos, sin = np.cos(ang), np.sin(ang)
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    if layout == ROPE_INTERLEAVED:
        x0, x1 = x[..., 0::2], x[..., 1::2]
        out[..., 0::2] = x0 * cos - x1 * sin
        out[..., 1::2] = x0 * sin + x1 * cos
    elif layout == ROPE_HALF:
        x0, x1 = x[..., : d // 2], x[..., d // 2:]
        out[..., : d // 2] = x0 * cos - x1 * sin
        out[..., d // 2:] = x1 * cos + x0 * sin
    else:
        raise ValueError(f"unknown RoPE layout {layout}")
    return out


# ---------------------------------------------------------------------------
# Cache append: c = RMSNorm(W_DKV h), k_R = RoPE(W_KR h)
# ---------------------------------------------------------------------------

def rms_norm(x, gamma, eps: float) -> np.ndarray:
    """gamma * x / sqrt(mean(x^2) + eps) over the last axis.

    "Hands-on DeepSeek MLA" (RMSNorm class: variance = mean(x^2), eps 1e-6,
    weight initialised to ones); "构建DeepSeek-V3：多头潜在注意力(MLA)架构"
    step 1, c_KV = RMSNorm(W_dkv x).
    """
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return _f64(gamma) * x / np.sqrt(ms + eps)


def latent_row(h, W_DKV, W_KR, gamma, pos, dims: Dims) -> np.ndarray:
    """The cache row ``[c ; k_R]`` one new token appends.

    c = RMSNorm(W_DKV h) and k_R = RoPE_pos(W_KR h), stored already rotated
    and shared by all heads: "解耦 RoPE（MLA 下）" §3.3-3.4 and §五 steps 2-3;
    "从零理解 MLA", 解耦 RoPE (k_t^R = RoPE(W^KR h_t)) and ``absorbed_step``
    (the row is ``cat([c_kv, k_r])``, c first).  ``h`` is ``[B, d_model]``,
    weights are ``[out, in]``; returns ``[B, d_c + d_rope]``.
    """
    h = _f64(h)
    x = h @ _f64(W_DKV).T
    c = rms_norm(x, gamma, dims.rms_eps)
    k = rope(h @ _f64(W_KR).T, _f64(pos), dims.rope_base, dims.rope_layout)
    return np.concatenate([c, k], axis=-1)


# ---------------------------------------------------------------------------
# 8-bit latent rows: c as int8 codes times a power-of-two scale
# ---------------------------------------------------------------------------

INT8_MAX = 127


def quantize_int8_pow2(c):
    """Per-row int8 quantisation with a power-of-two scale.

    "DeepSeek-V3多头潜在注意力(MLA)架构", 多头潜在注意力与KV缓存优化: the KV
    cache may be stored at lower precision (INT8 or INT4), at some cost in
    accuracy.  Reading taken here: each cached latent row c (d_c values) is
    stored as int8 codes q and one scale s = 2**e, the smallest power of two
    with max|c| / s <= 127, q = round-half-even(c / s); the row then reads back
    as q * s.  (A power-of-two scale keeps c / s and q * s exact, at the cost of
    at most one bit of the code range.)  An all-zero row gets e = 0.

    ``c [..., d_c]`` -> ``q [..., d_c]`` (int64 codes in [-127, 127]), ``e [...]``.
    """
    c = _f64(c)
    amax = np.abs(c).max(axis=-1)
    e = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    e[nz] = np.ceil(np.log2(amax[nz] / INT8_MAX)).astype(np.int64)
    s = np.exp2(e.astype(np.float64))[..., None]
    q = np.round(c / s)           # numpy rounds half to even
    return q.astype(np.int64), e


def dequantize_int8_pow2(q, e):
    """q * 2**e: the latent values an int8 row holds."""
    return _f64(q) * np.exp2(_f64(e))[..., None]


# ---------------------------------------------------------------------------
# Queries and absorption
# ---------------------------------------------------------------------------

def queries(x, W_DQ, W_UQ, W_QR, pos, dims: Dims):
    """Content and position queries of the new token.

    c_Q = W_DQ h when the query is compressed ("从零理解 MLA", 查询压缩), else
    c_Q = h ("解耦 RoPE（MLA 下）" §七 computes both from h).  Then
    q_C = W_UQ c_Q split into heads and q_R,i = RoPE_pos(W_QR,i c_Q)
    ("从零理解 MLA", 解耦 RoPE).  Returns ``q_C [B,H,d_nope]``, ``q_R [B,H,d_rope]``.
    """
    x = _f64(x)
    B = x.shape[0]
    H = dims.n_heads
    c_q = x @ _f64(W_DQ).T if W_DQ is not None else x
    q_c = (c_q @ _f64(W_UQ).T).reshape(B, H, dims.d_nope)
    q_r = (c_q @ _f64(W_QR).T).reshape(B, H, dims.d_rope)
    q_r = rope(q_r, _f64(pos)[:, None], dims.rope_base, dims.rope_layout)
    return q_c, q_r


def absorb_q(x, W_DQ, W_UQ, W_QR, W_UK, pos, dims: Dims) -> np.ndarray:
    """q_lat_i = [W_UK,i^T q_C,i ; q_R,i], shape ``[B, H, d_c + d_rope]``.

    The content query is folded through the per-head key up-projection so that
    the score is taken against the cached latent directly: "从零理解 MLA",
    矩阵吸收 ((W_i^UK)^T q_{t,i}^C dotted with c_j); "解耦 RoPE（MLA 下）" §五
    step 4.  W_UK is ``[H * d_nope, d_c]`` viewed ``[H, d_nope, d_c]``.
    """
    q_c, q_r = queries(x, W_DQ, W_UQ, W_QR, pos, dims)
    w_uk = _f64(W_UK).reshape(dims.n_heads, dims.d_nope, dims.d_c)
    q_tilde = np.einsum("bha,hac->bhc", q_c, w_uk)
    return np.concatenate([q_tilde, q_r], axis=-1)


# ---------------------------------------------------------------------------
# Attention over the cache
# ---------------------------------------------------------------------------

def attend_latent(q_lat, rows, dims: Dims):
    """Decode attention of one sequence in latent space.

    logits_{i,s} = scale * q_lat_i . row_s  (= q~_i . c_s + q_R,i . k_R,s),
    alpha = softmax over s, z_i = sum_s alpha_{i,s} c_s, and
    lse_i = log sum_s exp(logits_{i,s}).
    "从零理解 MLA", 解耦 RoPE ``absorbed_step`` (s_c + s_r, scale, softmax,
    z = attn . c_cache); "解耦 RoPE（MLA 下）" §五 steps 4-5.  The decode query
    sees every row it is given (its own row included).

    ``q_lat [H, d_c + d_rope]``, ``rows [L, d_c + d_rope]`` -> ``z [H, d_c]``,
    ``lse [H]``.  L = 0 gives z = 0 and lse = -inf.
    """
    q = _f64(q_lat)
    r = _f64(rows)
    H = q.shape[0]
    if r.shape[0] == 0:
        return np.zeros((H, dims.d_c)), np.full(H, -np.inf)
    logits = (q @ r.T) * dims.scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    z = (p @ r[:, : dims.d_c]) / l
    return z, (m + np.log(l))[:, 0]


def attend_unabsorbed(q_c, q_r, rows, W_UK, W_UV, dims: Dims):
    """Standard attention with K and V rebuilt from the cache (no absorption).

    K_{i,s} = [W_UK,i c_s ; k_R,s] (k_R copied to every head), V_{i,s} =
    W_UV,i c_s, score = q_i . K_{i,s} * scale, softmax, o_i = sum alpha V:
    "解耦 RoPE（MLA 下）" §七 ``forward_naive``; "从零理解 MLA", 解耦 RoPE
    ``MLADecoupledRoPE.forward``.

    ``q_c [H,d_nope]``, ``q_r [H,d_rope]``, ``rows [L, d_c + d_rope]`` ->
    ``o [H, d_v]``, ``alpha [H, L]``.
    """
    H = dims.n_heads
    r = _f64(rows)
    c, k_r = r[:, : dims.d_c], r[:, dims.d_c:]
    w_uk = _f64(W_UK).reshape(H, dims.d_nope, dims.d_c)
    w_uv = _f64(W_UV).reshape(H, dims.d_v, dims.d_c)
    k_c = np.einsum("hac,sc->hsa", w_uk, c)
    v = np.einsum("hvc,sc->hsv", w_uv, c)
    k = np.concatenate([k_c, np.broadcast_to(k_r, (H,) + k_r.shape)], axis=-1)
    q = np.concatenate([_f64(q_c), _f64(q_r)], axis=-1)
    logits = np.einsum("ha,hsa->hs", q, k) * dims.scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    alpha = p / p.sum(axis=1, keepdims=True)
    return np.einsum("hs,hsv->hv", alpha, v), alpha


def split_partial(q_lat, rows, dims: Dims):
    """One split of a split-KV pass: unnormalised (O_j, m_j, l_j).

    m_j = max_s logits, l_j = sum_s exp(logits - m_j),
    O_j = sum_s exp(logits - m_j) c_s over the rows of this split only.  The
    split-KV decomposition is the standard rewriting of one softmax as a
    weighted merge of partial softmaxes; with a single split,
    O/l and m + log l are exactly ``attend_latent``'s z and lse.
    """
    q = _f64(q_lat)
    r = _f64(rows)
    logits = (q @ r.T) * dims.scale
    m = logits.max(axis=1)
    p = np.exp(logits - m[:, None])
    return p @ r[:, : dims.d_c], m, p.sum(axis=1)


def combine_splits(O_parts, m_parts, l_parts):
    """Merge split-KV partials: z = sum_j w_j O_j / sum_j w_j l_j,
    w_j = exp(m_j - max_j m_j); lse = max m + log sum_j w_j l_j.

    ``O_parts [S, H, d_c]``, ``m_parts, l_parts [S, H]``.
    """
    O = _f64(O_parts)
    m = _f64(m_parts)
    l = _f64(l_parts)
    M = m.max(axis=0)
    w = np.exp(m - M[None])
    den = (w * l).sum(axis=0)
    z = (w[..., None] * O).sum(axis=0) / den[:, None]
    return z, M + np.log(den)


def unabsorb(z, W_UV, W_O, dims: Dims):
    """o_i = W_UV,i z_i, then optionally u = W_O concat_i(o_i).

    "从零理解 MLA", 矩阵吸收 (value side: aggregate in latent space, then one
    up-projection) and ``absorbed_step`` (o = einsum(z, w_uv), then w_o);
    "解耦 RoPE（MLA 下）" §七 ``forward_absorbed``.  ``z [B, H, d_c]``;
    W_UV ``[H * d_v, d_c]``; W_O ``[d_model, H * d_v]`` or None.
    Returns ``o [B, H * d_v]`` and ``u [B, d_model]`` (None without W_O).
    """
    z = _f64(z)
    B = z.shape[0]
    w_uv = _f64(W_UV).reshape(dims.n_heads, dims.d_v, dims.d_c)
    o = np.einsum("bhc,hvc->bhv", z, w_uv).reshape(B, dims.n_heads * dims.d_v)
    u = o @ _f64(W_O).T if W_O is not None else None
    return o, u


# ---------------------------------------------------------------------------
# Whole decode step and whole-sequence forward
# ---------------------------------------------------------------------------

def gather_rows(pool, block_table, b: int, length: int, page_size: int) -> np.ndarray:
    """Rows 0..length-1 of sequence b from a paged pool ``[pages, page_size, row]``.

    Row s lives in page ``block_table[b][s // page_size]`` at slot
    ``s % page_size`` (the paged-cache layout; the pages only say the cache
    is appended to and read whole, "从零理解 MLA", KV Cache).
    """
    idx = np.arange(length)
    pages = np.asarray(block_table)[b][idx // page_size]
    return _f64(np.asarray(pool)[pages, idx % page_size])


def decode_step(h, prior_rows, W, dims: Dims, unabsorbed: bool = True):
    """One decode step of a batch, written as the pages define it.

    Order per "解耦 RoPE（MLA 下）" §五: (2-3) append the new token's row,
    (4) queries, (5) attend over every cached row including the new one, then
    the output projections.  ``prior_rows[b]`` holds the rows already cached
    for sequence b (``[L_b - 1, d_c + d_rope]``); the new token sits at
    position ``pos_b = L_b - 1`` (0-based, "解耦 RoPE（MLA 下）" §4.3).

    ``W`` maps names to weights: W_DKV, W_KR, gamma, W_DQ (None for no query
    compression), W_UQ, W_QR, W_UK, W_UV, W_O (None to stop at o).
    With ``unabsorbed`` the attention runs in the un-absorbed form (K and V
    rebuilt per head); otherwise in latent space.  Returns a dict with
    ``row``, ``q_lat``, ``z``, ``lse``, ``o``, ``u``.
    """
    h = _f64(h)
    B = h.shape[0]
    pos = np.array([len(r) for r in prior_rows], dtype=np.int64)
    row = latent_row(h, W["W_DKV"], W["W_KR"], W["gamma"], pos, dims)
    q_c, q_r = queries(h, W.get("W_DQ"), W["W_UQ"], W["W_QR"], pos, dims)
    q_lat = absorb_q(h, W.get("W_DQ"), W["W_UQ"], W["W_QR"], W["W_UK"], pos, dims)
    zs, lses, os_ = [], [], []
    for b in range(B):
        rows = np.concatenate([_f64(prior_rows[b]).reshape(-1, dims.row), row[b:b + 1]], axis=0)
        z, lse = attend_latent(q_lat[b], rows, dims)
        zs.append(z)
        lses.append(lse)
        if unabsorbed:
            o_b, _ = attend_unabsorbed(q_c[b], q_r[b], rows, W["W_UK"], W["W_UV"], dims)
            os_.append(o_b.reshape(-1))
    z = np.stack(zs)
    if unabsorbed:
        o = np.stack(os_)
        u = o @ _f64(W["W_O"]).T if W.get("W_O") is not None else None
    else:
        o, u = unabsorb(z, W["W_UV"], W.get("W_O"), dims)
    return {"row": row, "q_lat": q_lat, "z": z, "lse": np.stack(lses), "o": o, "u": u}


def forward_naive(h_seq, W, dims: Dims) -> np.ndarray:
    """Whole-sequence causal MLA forward, K and V rebuilt (training / prefill form).

    "解耦 RoPE（MLA 下）" §七 ``forward_naive`` and "从零理解 MLA", 解耦 RoPE
    ``MLADecoupledRoPE.forward``: token t attends to tokens 0..t.
    ``h_seq [T, d_model]`` -> ``u [T, d_model]`` (or ``o [T, H*d_v]`` without W_O).
    """
    h = _f64(h_seq)
    T = h.shape[0]
    pos = np.arange(T)
    rows = latent_row(h, W["W_DKV"], W["W_KR"], W["gamma"], pos, dims)
    q_c, q_r = queries(h, W.get("W_DQ"), W["W_UQ"], W["W_QR"], pos, dims)
    outs = []
    for t in range(T):
        o_t, _ = attend_unabsorbed(q_c[t], q_r[t], rows[: t + 1], W["W_UK"], W["W_UV"], dims)
        outs.append(o_t.reshape(-1))
    o = np.stack(outs)
    return o @ _f64(W["W_O"]).T if W.get("W_O") is not None else o


def absorbed_decode_loop(h_seq, W, dims: Dims) -> np.ndarray:
    """Token-by-token absorbed decode of a sequence from an empty cache.

    "从零理解 MLA", 解耦 RoPE: ``absorbed_step`` called for t = 0..L-1, each
    step appending its row and attending over the cache in latent space; its
    outputs equal ``forward_naive`` row by row.
    """
    h = _f64(h_seq)
    rows = np.zeros((0, dims.row))
    outs = []
    for t in range(h.shape[0]):
        step = decode_step(h[t:t + 1], [rows], W, dims, unabsorbed=False)
        rows = np.concatenate([rows, step["row"]], axis=0)
        outs.append((step["u"] if step["u"] is not None else step["o"])[0])
    return np.stack(outs)
