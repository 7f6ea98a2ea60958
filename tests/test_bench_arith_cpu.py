"""The bench's roofline denominators, checked against the method's sizes.

The roofline fraction bench.py prints is algorithmic work / time, so a wrong
byte or FLOP count would misreport every kernel.  These tests recount the work
from the DeepSeek-V2 dimensions ("从零理解 MLA", 实际配置: 128 heads, d_c 512,
d_R 64, d_nope = d_v = 128, d_model 5120, q_lora 1536) and the cache row of
the absorbed form (c and k_R, 576 values per cached token) and compare with
bench.algorithmic() for the benched workloads.
"""

import numpy as np
import pytest

import bench
from mla_latent_kv_45_b200 import synth

H, D_C, D_R, D_NOPE, D_V, D_MODEL, D_Q = 128, 512, 64, 128, 128, 5120, 1536


def v2_params():
    # W_DKV, W_KR (append); W_DQ, W_UQ, W_QR, W_UK (absorption); W_UV, W_O
    return (D_C * D_MODEL + D_R * D_MODEL + D_Q * D_MODEL + H * D_NOPE * D_Q + H * D_R * D_Q
            + H * D_NOPE * D_C + H * D_V * D_C + D_MODEL * H * D_V)


def test_v2_parameter_count():
    assert v2_params() == 149_225_472


@pytest.mark.parametrize("name", ["v2_batch64", "v2_step128", "v2_single"])
def test_decode_step_work(name):
    wl = synth.WORKLOADS[name]
    prior = synth.make_prior_lengths(wl)
    lens = bench.attended_lengths(wl, prior)
    got = bench.algorithmic(wl, lens)
    B = wl.batch
    rows = int((prior + 1).sum())          # every cached row and the appended one
    # per cached row: 576 bf16 values read once; per row and head: the score
    # (2 x 576) and its share of z (2 x 512)
    attn_bytes = rows * 576 * 2 + B * H * (576 + 512) * 2
    attn_flops = rows * H * (2 * 576 + 2 * 512)
    # weights once, the appended rows written, h read and the layer output written
    step_bytes = attn_bytes + 2 * v2_params() + B * 576 * 2 + 2 * B * D_MODEL * 2
    step_flops = attn_flops + 2 * B * v2_params()
    assert got["rows"] == rows
    assert got["attn_bytes"] == attn_bytes
    assert got["attn_flops"] == attn_flops
    assert got["step_bytes"] == step_bytes
    assert got["step_flops"] == step_flops


def test_headline_figures():
    """The figures the measured-status tables quote for the batch-64 workload."""
    wl = synth.WORKLOADS["v2_batch64"]
    got = bench.algorithmic(wl, bench.attended_lengths(wl, synth.make_prior_lengths(wl)))
    assert got["attn_bytes"] == 329_730_944
    assert got["attn_flops"] == 75_411_734_528
    assert got["step_bytes"] == 629_566_336


def test_long_context_attention_only():
    wl = synth.WORKLOADS["v2_long"]
    prior = synth.make_prior_lengths(wl)
    lens = bench.attended_lengths(wl, prior)
    got = bench.algorithmic(wl, lens)
    rows = int(lens.sum())
    assert rows == 8 * 131_072
    assert got["attn_bytes"] == rows * 1152 + 8 * H * (576 + 512) * 2
    assert got["step_bytes"] == got["attn_bytes"]       # attention alone


def test_int8_rows_cost_656_bytes():
    wl = synth.WORKLOADS["v2_batch64_int8"]
    prior = synth.make_prior_lengths(wl)
    got = bench.algorithmic(wl, bench.attended_lengths(wl, prior))
    rows = int((prior + 1).sum())
    assert got["attn_bytes"] == rows * 656 + wl.batch * H * (576 + 512) * 2


def test_prefill_chunk_reads_each_row_once():
    """A chunk's T entries share their sequence's rows: the bytes count each
    cached row once, the FLOPs count every (token, row) pair of the causal mask."""
    wl = synth.WORKLOADS["v2_prefill256"]
    prior = synth.make_prior_lengths(wl)
    lens = bench.attended_lengths(wl, prior)
    got = bench.algorithmic(wl, lens)
    T = wl.new_tokens
    assert len(lens) == wl.batch * T
    assert np.array_equal(lens, np.concatenate([p + 1 + np.arange(T) for p in prior]))
    cached = wl.batch * (wl.prior_max + T)
    assert got["attn_bytes"] == cached * 1152 + wl.batch * T * H * (576 + 512) * 2
    assert got["attn_flops"] == int(lens.sum()) * H * 2176


def test_measured_peaks_file_layouts(tmp_path):
    """The roofline's denominators come from MEASURED_PEAKS.json when it holds
    them, at any depth of the file; anything else falls back, never fails."""
    import json
    flat = tmp_path / "flat.json"
    flat.write_text(json.dumps({"hbm_gbs": 6542.1, "bf16_tflops": 1641.8,
                                "bf16_tflops_sustained": 1367.1}))
    assert bench.peaks(str(flat)) == (6542.1, 1641.8, 1367.1, "measured")
    nested = tmp_path / "nested.json"
    nested.write_text(json.dumps({"gpu": "B200", "peaks": {"hbm_gbs": 6500, "bf16_tflops": 1600}}))
    hbm, tf, sus, src = bench.peaks(str(nested))
    assert (hbm, tf, sus, src) == (6500.0, 1600.0, None, "measured")
    missing = tmp_path / "missing.json"
    missing.write_text(json.dumps({"hbm_gbs": 6500}))
    assert bench.peaks(str(missing))[3] == "fallback"
    broken = tmp_path / "broken.json"
    broken.write_text("{not json")
    assert bench.peaks(str(broken))[3] == "fallback"
    assert bench.peaks(str(tmp_path / "absent.json"))[3] == "fallback"
