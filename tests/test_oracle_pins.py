"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every check is written as ``check_*(fn)`` and run on the oracle (must pass);
the ``test_pins_catch_*`` tests run the same checks on oracle copies with a
planted mistake (a dropped term, a flipped sign, a swapped operand) and
require them to fail, so a plausible slip in the oracle cannot go unnoticed.
No value here comes from the CUDA path.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from oracle.mla_oracle import (Dims, ROPE_HALF, ROPE_INTERLEAVED, absorb_q, attend_latent,
                               attend_unabsorbed, combine_splits, latent_row, queries,
                               rms_norm, rope, split_partial, unabsorb)

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


@pytest.fixture(scope="module")
def hand():
    with open(GOLD, encoding="utf-8") as f:
        return json.load(f)


def _r(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# P1: the pages' hand-worked example (解耦 RoPE（MLA 下） §四)
# ---------------------------------------------------------------------------

def check_hand_k_rows(hand, rope_fn):
    Hm = np.array(hand["H"], float)
    wkr = np.array(hand["W_KR"], float)
    k0 = Hm @ wkr.T
    assert np.array_equal(k0, np.array(hand["k_R_unrotated"], float))
    k = rope_fn(k0, np.array(hand["positions"], float), 10000.0, ROPE_INTERLEAVED)
    np.testing.assert_allclose(k, hand["k_R_cached"], atol=0.5e-3)
    t = np.array(hand["positions"], float)
    np.testing.assert_allclose(k, np.stack([np.cos(t), np.sin(t)], 1), atol=1e-15)


def check_hand_scores(hand, rope_fn):
    pos_q = hand["positions"][-1]
    q = rope_fn(np.array(hand["q_R_unrotated"], float), pos_q, 10000.0, ROPE_INTERLEAVED)
    np.testing.assert_allclose(q, hand["q_R_rotated"], atol=0.5e-3)
    k0 = np.array(hand["k_R_unrotated"], float)
    for shift in (0, hand["shift"]):
        t = np.array(hand["positions"], float) + shift
        k = rope_fn(k0, t, 10000.0, ROPE_INTERLEAVED)
        qq = rope_fn(np.array(hand["q_R_unrotated"], float), pos_q + shift, 10000.0,
                     ROPE_INTERLEAVED)
        ps = qq @ k.T
        np.testing.assert_allclose(ps, hand["position_scores"], atol=0.5e-3)
        # cos(s - t) for head 1, sin(s - t) for head 2 (§4.5)
        d = np.array(hand["positions"], float) - pos_q
        np.testing.assert_allclose(ps[0], np.cos(d), atol=1e-14)
        np.testing.assert_allclose(ps[1], np.sin(d), atol=1e-14)
        tot = np.array(hand["content_scores"], float) + ps
        np.testing.assert_allclose(tot, hand["total_scores"], atol=1.01e-3)


def test_hand_example_k_rows(hand):
    check_hand_k_rows(hand, rope)


def test_hand_example_scores_and_shift(hand):
    check_hand_scores(hand, rope)


def test_hand_example_through_latent_row(hand):
    """latent_row's k_R half reproduces the cached position rows (§4.2-4.3)."""
    Hm = np.array(hand["H"], float)
    dims = Dims(n_heads=2, d_c=2, d_rope=2, d_nope=2, d_v=2)
    W_DKV = _r(0).standard_normal((2, 4))
    rows = latent_row(Hm, W_DKV, np.array(hand["W_KR"], float), np.ones(2), np.arange(3), dims)
    np.testing.assert_allclose(rows[:, 2:], hand["k_R_cached"], atol=0.5e-3)


def test_hand_example_concat(hand):
    """Concatenated dot product equals the sum of the two parts (§4.6)."""
    cc = hand["concat_check"]
    assert abs(np.dot(cc["q"], cc["k"]) - cc["dot"]) < 1e-12


def test_hand_example_attention_totals(hand):
    """attend_latent with scale 1 sees logits = content + position (§4.6 totals).

    The latent rows c_猫 = e1, c_吃 = e2, c_鱼 = (e1 + e2)/2 with q~_1 = e1,
    q~_2 = e2 reproduce the given content scores; the position half uses the
    page's own q_R and k_R.  z and lse must then be the softmax of the printed
    totals (rounded to 3 decimals on the page).
    """
    c = np.array([[1, 0], [0, 1], [0.5, 0.5]], float)
    k = np.array(hand["k_R_cached"], float)
    rows = np.concatenate([c, k], axis=1)
    q = np.concatenate([np.eye(2), np.array(hand["q_R_unrotated"], float)], axis=1)
    q[:, 2:] = rope(q[:, 2:], 2, 10000.0, ROPE_INTERLEAVED)
    dims = Dims(n_heads=2, d_c=2, d_rope=2, d_nope=2, d_v=2, softmax_scale=1.0)
    z, lse = attend_latent(q, rows, dims)
    tot = np.array(hand["total_scores"], float)
    w = np.exp(tot - tot.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    np.testing.assert_allclose(z, w @ c, atol=2e-3)
    np.testing.assert_allclose(lse, np.log(np.exp(tot).sum(1)), atol=2e-3)


# ---------------------------------------------------------------------------
# P2: RoPE -- relative-position identity, library routines, group laws
# ---------------------------------------------------------------------------

def check_rope_relative(rope_fn, layout):
    g = _r(1)
    for d in (2, 8, 64):
        q, k = g.standard_normal(d), g.standard_normal(d)
        for t, s in ((0, 0), (3, 11), (1000, 7), (131071, 5)):
            lhs = rope_fn(q, t, 10000.0, layout) @ rope_fn(k, s, 10000.0, layout)
            rhs = q @ rope_fn(k, s - t, 10000.0, layout)
            assert abs(lhs - rhs) < 1e-9 * (1 + abs(lhs)), (d, t, s)


def check_rope_gptj(rope_fn):
    """Interleaved pairing equals GPT-J's rotary embedding (library routine)."""
    from transformers.models.gptj import modeling_gptj as mg
    d, P = 64, 48
    x = _r(2).standard_normal((1, P, 1, d))
    sincos = mg.create_sinusoidal_positions(P, d).double()          # [P, d] = [sin | cos]
    sin, cos = sincos[None, :, : d // 2], sincos[None, :, d // 2:]
    ref = mg.apply_rotary_pos_emb(torch.from_numpy(x), sin, cos).numpy()
    got = rope_fn(x, np.arange(P)[None, :, None], 10000.0, ROPE_INTERLEAVED)
    np.testing.assert_allclose(got, ref, atol=2e-5)


def check_rope_llama(rope_fn):
    """Half-split pairing equals LLaMA's rotate_half embedding (library routine)."""
    from transformers.models.gptj import modeling_gptj as mg
    from transformers.models.llama import modeling_llama as ml
    d, P = 64, 48
    x = _r(3).standard_normal((1, 1, P, d))
    sincos = mg.create_sinusoidal_positions(P, d).double()
    sin, cos = sincos[:, : d // 2], sincos[:, d // 2:]
    cos2 = torch.cat([cos, cos], -1)[None]
    sin2 = torch.cat([sin, sin], -1)[None]
    ref, _ = ml.apply_rotary_pos_emb(torch.from_numpy(x), torch.from_numpy(x), cos2, sin2)
    got = rope_fn(x, np.arange(P)[None, None, :], 10000.0, ROPE_HALF)
    np.testing.assert_allclose(got, ref.numpy(), atol=2e-5)


def test_rope_relative_identity():
    check_rope_relative(rope, ROPE_INTERLEAVED)
    check_rope_relative(rope, ROPE_HALF)


def test_rope_matches_gptj():
    check_rope_gptj(rope)


def test_rope_matches_llama():
    check_rope_llama(rope)


def test_rope_group_laws():
    g = _r(4)
    for layout in (ROPE_INTERLEAVED, ROPE_HALF):
        x = g.standard_normal((5, 64))
        np.testing.assert_allclose(rope(x, 0, 1e4, layout), x, atol=0)
        a, b = 37.0, 1234.0
        np.testing.assert_allclose(rope(rope(x, a, 1e4, layout), b, 1e4, layout),
                                   rope(x, a + b, 1e4, layout), atol=1e-10)
        np.testing.assert_allclose(np.linalg.norm(rope(x, 99, 1e4, layout), axis=1),
                                   np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_layouts_are_a_permutation():
    """Half-split RoPE is interleaved RoPE on re-paired coordinates."""
    d = 64
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])  # half index -> interleaved
    x_half = _r(5).standard_normal(d)
    x_int = np.empty(d)
    x_int[perm] = x_half
    got = rope(x_half, 321, 1e4, ROPE_HALF)
    ref = rope(x_int, 321, 1e4, ROPE_INTERLEAVED)[perm]
    np.testing.assert_allclose(got, ref, atol=1e-14)


# ---------------------------------------------------------------------------
# P5: RMSNorm closed forms and the library routine
# ---------------------------------------------------------------------------

def check_rmsnorm(fn):
    g = _r(6)
    x = g.standard_normal((7, 512)) * 3.0
    gamma = 1 + 0.1 * g.standard_normal(512)
    eps = 1e-6
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (512,), torch.from_numpy(gamma), eps)
    np.testing.assert_allclose(fn(x, gamma, eps), ref.numpy(), rtol=1e-12, atol=1e-12)
    ms = (x * x).mean(1)
    out = fn(x, np.ones(512), eps)
    np.testing.assert_allclose(np.sqrt((out * out).mean(1)), np.sqrt(ms / (ms + eps)), rtol=1e-12)
    np.testing.assert_allclose(fn(1e3 * x, gamma, 0.0), fn(x, gamma, 0.0), rtol=1e-12)


def test_rmsnorm_pins():
    check_rmsnorm(rms_norm)


# ---------------------------------------------------------------------------
# P3: absorption identity at the pages' toy shapes
# ---------------------------------------------------------------------------

TOY_P1 = dict(d_model=64, n_heads=4, d_c=8, d_rope=4, d_nope=16, d_v=16, d_q=0)     # 解耦 RoPE §七
TOY_P3 = dict(d_model=128, n_heads=4, d_c=32, d_rope=8, d_nope=16, d_v=16, d_q=48)  # 从零理解 MLA


def toy_weights(cfg, seed, layout=ROPE_INTERLEAVED, with_o=True):
    g = _r(seed)
    H, dm = cfg["n_heads"], cfg["d_model"]
    dq_in = cfg["d_q"] or dm
    W = {
        "W_DKV": g.standard_normal((cfg["d_c"], dm)) * 0.2,
        "W_KR": g.standard_normal((cfg["d_rope"], dm)) * 0.2,
        "gamma": 1 + 0.1 * g.standard_normal(cfg["d_c"]),
        "W_DQ": g.standard_normal((cfg["d_q"], dm)) * 0.2 if cfg["d_q"] else None,
        "W_UQ": g.standard_normal((H * cfg["d_nope"], dq_in)) * 0.2,
        "W_QR": g.standard_normal((H * cfg["d_rope"], dq_in)) * 0.2,
        "W_UK": g.standard_normal((H * cfg["d_nope"], cfg["d_c"])) * 0.2,
        "W_UV": g.standard_normal((H * cfg["d_v"], cfg["d_c"])) * 0.2,
        "W_O": g.standard_normal((dm, H * cfg["d_v"])) * 0.2 if with_o else None,
    }
    dims = Dims(n_heads=H, d_c=cfg["d_c"], d_rope=cfg["d_rope"], d_nope=cfg["d_nope"],
                d_v=cfg["d_v"], rope_layout=layout)
    return W, dims


def check_absorption(absorb_fn, attend_fn, unabsorb_fn):
    for cfg, seed in ((TOY_P1, 10), (TOY_P3, 11)):
        for layout in (ROPE_INTERLEAVED, ROPE_HALF):
            W, dims = toy_weights(cfg, seed, layout)
            g = _r(seed + 100)
            L = 10
            rows = g.standard_normal((L, dims.row))
            h = g.standard_normal((3, cfg["d_model"]))
            pos = np.array([9, 4, 0])
            q_c, q_r = queries(h, W["W_DQ"], W["W_UQ"], W["W_QR"], pos, dims)
            q_lat = absorb_fn(h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], pos, dims)
            for b in range(3):
                o_ref, alpha = attend_unabsorbed(q_c[b], q_r[b], rows, W["W_UK"], W["W_UV"], dims)
                z, _ = attend_fn(q_lat[b], rows, dims)
                # absorbed logits == un-absorbed logits -> identical weights
                lg = (q_lat[b] @ rows.T) * dims.scale
                a2 = np.exp(lg - lg.max(1, keepdims=True))
                a2 /= a2.sum(1, keepdims=True)
                np.testing.assert_allclose(a2, alpha, rtol=1e-12, atol=1e-14)
                o, _ = unabsorb_fn(z[None], W["W_UV"], None, dims)
                np.testing.assert_allclose(o[0], o_ref.reshape(-1), rtol=1e-10, atol=1e-12)


def test_absorption_identity():
    check_absorption(absorb_q, attend_latent, unabsorb)


def check_naive_equals_absorbed(naive_fn, loop_fn):
    for cfg, seed in ((TOY_P1, 20), (TOY_P3, 21)):
        W, dims = toy_weights(cfg, seed)
        h = _r(seed).standard_normal((10, cfg["d_model"]))
        a = naive_fn(h, W, dims)
        b = loop_fn(h, W, dims)
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_naive_forward_equals_absorbed_decode_loop():
    """The pages' equivalence test (解耦 RoPE §七; 从零理解 MLA, 解耦 RoPE), our seeds."""
    check_naive_equals_absorbed(oracle.forward_naive, oracle.absorbed_decode_loop)


# ---------------------------------------------------------------------------
# P4: special cases that reduce to textbook / library routines
# ---------------------------------------------------------------------------

def check_attend_special(attend_fn):
    g = _r(30)
    dims = Dims(n_heads=4, d_c=16, d_rope=8, d_nope=8, d_v=8)
    rows = g.standard_normal((37, dims.row))
    q = g.standard_normal((4, dims.row))
    # one row: z is that row's latent exactly
    z, lse = attend_fn(q, rows[:1], dims)
    np.testing.assert_allclose(z, np.broadcast_to(rows[0, :16], (4, 16)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, (q @ rows[0]) * dims.scale, rtol=1e-14)
    # equal scores: mean of the latents
    z, lse = attend_fn(np.zeros_like(q), rows, dims)
    np.testing.assert_allclose(z, np.broadcast_to(rows[:, :16].mean(0), (4, 16)), atol=1e-14)
    np.testing.assert_allclose(lse, np.log(37.0), rtol=1e-14)
    # one dominant score
    q2 = 1e4 * rows[5] / np.linalg.norm(rows[5]) ** 2 / dims.scale
    z, _ = attend_fn(np.broadcast_to(q2, (4, dims.row)).copy(), rows, dims)
    assert np.abs(z - rows[5, :16]).max() < 1e-6
    # plain MQA attention (library SDPA): all heads share K = rows, V = latents
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(rows)[None, None].expand(1, 4, -1, -1),
        torch.from_numpy(rows[:, :16])[None, None].expand(1, 4, -1, -1), scale=dims.scale)
    z, lse = attend_fn(q, rows, dims)
    np.testing.assert_allclose(z, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(q @ rows.T) * dims.scale, 1),
                               rtol=1e-13)


def test_attend_special_cases():
    check_attend_special(attend_latent)


def test_unabsorbed_reduces_to_mqa():
    """W_UK,i = I, W_UV,i = I, no RoPE part: plain MQA with K = V = c (library SDPA)."""
    g = _r(31)
    d = 16
    dims = Dims(n_heads=3, d_c=d, d_rope=2, d_nope=d, d_v=d)
    c = g.standard_normal((20, d))
    rows = np.concatenate([c, np.zeros((20, 2))], 1)
    eye = np.tile(np.eye(d), (3, 1))
    q_c = g.standard_normal((3, d))
    o, _ = attend_unabsorbed(q_c, g.standard_normal((3, 2)), rows, eye, eye, dims)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q_c)[None, :, None], torch.from_numpy(c)[None, None].expand(1, 3, -1, -1),
        torch.from_numpy(c)[None, None].expand(1, 3, -1, -1), scale=dims.scale)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-14)


def test_split_combine():
    g = _r(32)
    dims = Dims(n_heads=4, d_c=16, d_rope=8, d_nope=8, d_v=8)
    rows = g.standard_normal((100, dims.row))
    q = 3 * g.standard_normal((4, dims.row))
    z_ref, lse_ref = attend_latent(q, rows, dims)
    O, m, l = split_partial(q, rows, dims)
    z, lse = combine_splits(O[None], m[None], l[None])
    np.testing.assert_allclose(z, z_ref, rtol=1e-14, atol=1e-15)
    for cuts in ([0, 1, 100], [0, 33, 34, 90, 100], list(range(0, 101, 10))):
        parts = [split_partial(q, rows[a:b], dims) for a, b in zip(cuts[:-1], cuts[1:])]
        z, lse = combine_splits(*[np.stack(p) for p in zip(*parts)])
        np.testing.assert_allclose(z, z_ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, lse_ref, rtol=1e-13)


def test_empty_sequence():
    dims = Dims(n_heads=2, d_c=4, d_rope=2, d_nope=2, d_v=2)
    z, lse = attend_latent(np.ones((2, 6)), np.zeros((0, 6)), dims)
    assert np.all(z == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------------------
# P6: brute force on tiny inputs
# ---------------------------------------------------------------------------

def check_brute(step_fn):
    for cfg, seed, layout in ((TOY_P1, 40, ROPE_INTERLEAVED), (TOY_P3, 41, ROPE_HALF)):
        cfg = dict(cfg, d_model=min(cfg["d_model"], 24))
        W, dims = toy_weights(cfg, seed, layout)
        g = _r(seed)
        h = g.standard_normal((2, cfg["d_model"]))
        prior = [g.standard_normal((5, dims.row)), g.standard_normal((2, dims.row))]
        got = step_fn(h, prior, W, dims)
        tolist = lambda a: None if a is None else np.asarray(a).tolist()
        Wl = {k: tolist(v) for k, v in W.items()}
        ref = brute.decode_step(h.tolist(), [p.tolist() for p in prior], Wl, dims.n_heads,
                                dims.d_c, dims.d_rope, dims.d_nope, dims.d_v, layout=layout)
        for b in range(2):
            row, q_lat, z, o, u = ref[b]
            np.testing.assert_allclose(got["row"][b], row, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(got["q_lat"][b], q_lat, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(got["z"][b], z, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(got["o"][b], o, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(got["u"][b], u, rtol=1e-11, atol=1e-12)


def test_brute_force_decode_step():
    check_brute(lambda h, p, W, d: oracle.decode_step(h, p, W, d, unabsorbed=True))
    check_brute(lambda h, p, W, d: oracle.decode_step(h, p, W, d, unabsorbed=False))


# ---------------------------------------------------------------------------
# bf16 rounding used for the cache-write comparison target
# ---------------------------------------------------------------------------

def test_bf16_round_matches_torch():
    g = _r(50)
    x = np.concatenate([g.standard_normal(10000).astype(np.float32),
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3e-39, 1e-40])])
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.bf16_round(x.astype(np.float64)), ref)


# ---------------------------------------------------------------------------
# The pins catch planted mistakes (mutants of oracle functions)
# ---------------------------------------------------------------------------

def _rope_sign_flip(x, pos, base=1e4, layout=0):
    return rope(x, -np.asarray(pos, float), base, layout)


def _rope_wrong_freq(x, pos, base=1e4, layout=0):
    x = np.asarray(x, float)
    d = x.shape[-1]
    ang = np.asarray(pos, float)[..., None] * base ** (-np.arange(d // 2) / d)   # drops the 2
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)))
    out[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    out[..., 1::2] = x[..., 0::2] * s + x[..., 1::2] * c
    return out


def _rope_half_as_interleaved(x, pos, base=1e4, layout=0):
    return rope(x, pos, base, ROPE_INTERLEAVED)


def _rms_no_eps(x, gamma, eps):
    return rms_norm(x, gamma, 0.0)


def _rms_gamma_dropped(x, gamma, eps):
    return rms_norm(x, np.ones_like(np.asarray(gamma, float)), eps)


def _absorb_transposed(x, W_DQ, W_UQ, W_QR, W_UK, pos, dims):
    d = dims.d_nope
    w = np.asarray(W_UK, float).reshape(dims.n_heads, d, dims.d_c)
    w = np.ascontiguousarray(np.roll(w, 1, axis=0)).reshape(-1, dims.d_c)   # wrong head
    return absorb_q(x, W_DQ, W_UQ, W_QR, w, pos, dims)


def _attend_no_rope_part(q, rows, dims):
    q = np.array(q, float)
    q[:, dims.d_c:] = 0
    return attend_latent(q, rows, dims)


def _attend_wrong_scale(q, rows, dims):
    return attend_latent(q, rows, Dims(dims.n_heads, dims.d_c, dims.d_rope, dims.d_nope,
                                       dims.d_v, softmax_scale=1 / math.sqrt(dims.d_nope)))


def _unabsorb_transposed(z, W_UV, W_O, dims):
    w = np.asarray(W_UV, float).reshape(dims.n_heads, dims.d_v, dims.d_c)
    w = np.roll(w, 1, axis=2).reshape(-1, dims.d_c)
    return unabsorb(z, w, W_O, dims)


def _fails(fn, *a):
    try:
        fn(*a)
    except AssertionError:
        return True
    return False


def test_pins_catch_rope_mistakes(hand):
    assert _fails(check_hand_scores, hand, _rope_sign_flip)
    assert _fails(check_rope_gptj, _rope_wrong_freq)
    assert _fails(check_rope_llama, _rope_half_as_interleaved)
    assert _fails(check_rope_relative, _rope_sign_flip, ROPE_INTERLEAVED) is False  # identity is sign-blind
    assert _fails(check_rope_gptj, _rope_sign_flip)


def test_pins_catch_rmsnorm_mistakes():
    assert _fails(check_rmsnorm, _rms_no_eps)
    assert _fails(check_rmsnorm, _rms_gamma_dropped)


def test_pins_catch_absorption_mistakes():
    assert _fails(check_absorption, _absorb_transposed, attend_latent, unabsorb)
    assert _fails(check_absorption, absorb_q, _attend_no_rope_part, unabsorb)
    assert _fails(check_absorption, absorb_q, attend_latent, _unabsorb_transposed)
    assert _fails(check_attend_special, _attend_wrong_scale)


# ---------------------------------------------------------------------------
# Paged-cache gather: row s of sequence b sits at page bt[b][s // P], slot s % P
# ---------------------------------------------------------------------------

def check_gather(gather_fn):
    """Scatter known rows into a shuffled pool one at a time (the layout's
    definition, written as a loop), then the gather must give them back in
    logical order, for ragged lengths and for a length that ends mid-page."""
    rng = _r(77)
    P, width, pages = 4, 5, 11
    perm = rng.permutation(pages)
    bt = np.full((2, 4), -1, dtype=np.int64)
    bt[0, :3] = perm[:3]
    bt[1, :4] = perm[3:7]
    pool = np.full((pages, P, width), np.nan)
    rows = {0: rng.standard_normal((10, width)), 1: rng.standard_normal((13, width))}
    for b, r in rows.items():
        for s in range(len(r)):
            pool[bt[b, s // P], s % P] = r[s]
    for b, r in rows.items():
        for n in (1, P, P + 1, len(r)):
            got = gather_fn(pool, bt, b, n, P)
            assert got.shape == (n, width)
            assert np.array_equal(got, r[:n])


def test_gather_rows_pin():
    check_gather(oracle.gather_rows)


def test_pins_catch_gather_mistakes():
    def slot_swapped(pool, bt, b, n, P):   # page and slot indices exchanged
        idx = np.arange(n)
        return np.asarray(pool)[np.asarray(bt)[b][idx % P], idx // P]

    def pool_order(pool, bt, b, n, P):     # ignores the page table
        return np.asarray(pool).reshape(-1, pool.shape[-1])[:n]

    for bad in (slot_swapped, pool_order):
        assert _fails(check_gather, bad)


# ---------------------------------------------------------------------------
# int8 latent rows (KV-cache quantisation, "DeepSeek-V3多头潜在注意力(MLA)架构",
# 多头潜在注意力与KV缓存优化): codes times a power-of-two scale
# ---------------------------------------------------------------------------

def check_int8(quant, dequant):
    rng = _r(91)
    c = rng.standard_normal((40, 512)) * np.exp2(rng.integers(-12, 12, size=(40, 1)))
    c[3] = 0.0
    q, e = quant(c)
    assert q.shape == c.shape and e.shape == (40,)
    assert np.all(np.abs(q) <= 127)
    s = np.exp2(e.astype(float))[:, None]
    # the tightest power of two: the largest code uses more than half the range
    nz = np.abs(c).max(1) > 0
    assert np.all(np.abs(q[nz]).max(1) >= 64)
    assert e[3] == 0 and np.all(q[3] == 0)
    # brute force over exponents: the smallest e with max|round(c / 2^e)| <= 127
    for i in np.flatnonzero(nz)[:8]:
        best = min(k for k in range(-40, 40)
                   if np.abs(np.round(c[i] / 2.0 ** k)).max() <= 127)
        assert e[i] == best
    # library rounding (half to even) of the scaled row, and the error bound
    assert np.array_equal(q, torch.round(torch.from_numpy(c / s)).numpy().astype(np.int64))
    d = dequant(q, e)
    assert np.all(np.abs(d - c) <= s / 2)
    # exact ties go to even codes
    t = np.array([[0.5, 1.5, 2.5, -0.5, -2.5, 127.0]])
    qt, et = quant(t)
    assert et[0] == 0 and qt[0].tolist() == [0, 2, 2, 0, -2, 127]


def test_int8_pins():
    check_int8(oracle.quantize_int8_pow2, oracle.dequantize_int8_pow2)


def test_pins_catch_int8_mistakes():
    def loose_scale(c):      # scale one power of two too large
        q, e = oracle.quantize_int8_pow2(c)
        e = e + 1
        return np.round(c / np.exp2(e.astype(float))[:, None]).astype(np.int64), e

    def truncating(c):       # rounds toward zero
        q, e = oracle.quantize_int8_pow2(c)
        return np.trunc(c / np.exp2(e.astype(float))[:, None]).astype(np.int64), e

    def half_up(c):          # rounds halves away from zero
        q, e = oracle.quantize_int8_pow2(c)
        x = c / np.exp2(e.astype(float))[:, None]
        return (np.sign(x) * np.floor(np.abs(x) + 0.5)).astype(np.int64), e

    for bad in (loose_scale, truncating, half_up):
        assert _fails(check_int8, bad, oracle.dequantize_int8_pow2)
