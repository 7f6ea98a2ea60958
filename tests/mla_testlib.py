"""Helpers shared by the GPU parity tests: moving seeded inputs to the device
and the tolerance measures.

Tolerances (bf16 inputs): max|g - r| <= 2e-2 and sum|g - r| / sum|r| <= 5e-3;
fp32 validation mode: max|g - r| / max|r| <= 1e-4.  The reference r is always
the fp64 oracle on the same stored inputs.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import synth

BF16_MAX_ABS = 2e-2
BF16_MEAN_REL = 5e-3
FP32_REL = 1e-4
# lse of the bf16 path: the kernels sum the bf16-rounded P values the MMA
# consumes, each within 2^-9 relative of the exact weight, so l may be off by a
# factor (1 + d), |d| <= 2^-9, and lse by ln(1 + 2^-9) = 1.95e-3, plus the
# approximate exp2 / log2 (~1e-6).  On top of that the raw scores are fp32 sums
# of 576 products accumulated by the tensor core in its own order; that error
# scales with the logits' size, hence a relative term (logits of ~50 nats in
# the rescale test showed 3.5e-3 in all).
LSE_ATOL = 3e-3
LSE_RTOL = 5e-5


def lib_dims(wl: synth.Workload, **kw) -> L.Dims:
    return L.Dims(wl.n_heads, wl.d_c, wl.d_rope, wl.d_nope, wl.d_v, wl.page_size,
                  L.MLA_BF16 if wl.dtype == "bf16" else L.MLA_FP32, wl.rope_layout, wl.rope_base,
                  wl.rms_eps, kw.get("softmax_scale", 0.0))


def oracle_dims(wl: synth.Workload, **kw) -> oracle.Dims:
    return oracle.Dims(n_heads=wl.n_heads, d_c=wl.d_c, d_rope=wl.d_rope, d_nope=wl.d_nope,
                       d_v=wl.d_v, rope_base=wl.rope_base, rms_eps=wl.rms_eps,
                       softmax_scale=kw.get("softmax_scale", 0.0), rope_layout=wl.rope_layout)


def tdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def dev(a, wl, device="cuda"):
    """float32 host array (values already representable) -> device tensor of the workload dtype."""
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).to(tdtype(wl))


def dev_weights(W: dict, wl) -> dict:
    return {k: dev(v, wl) for k, v in W.items()}


def dev_cache(pc: synth.PagedCache, seq_lens, device="cuda") -> L.PagedCache:
    if pc.pool.dtype == np.uint16:
        pool = torch.from_numpy(pc.pool.view(np.int16)).to(device).view(torch.bfloat16)
    else:
        pool = torch.from_numpy(pc.pool).to(device)
    bt = torch.from_numpy(np.ascontiguousarray(pc.block_table, dtype=np.int32)).to(device)
    lens = torch.from_numpy(np.asarray(seq_lens, dtype=np.int32)).to(device)
    return L.PagedCache(pool, bt, lens)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def metrics(g, r):
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    err = np.abs(g - r)
    return {"max_abs": float(err.max(initial=0.0)),
            "mean_rel": float(err.sum() / max(np.abs(r).sum(), 1e-300)),
            "rel": float(err.max(initial=0.0) / max(np.abs(r).max(initial=0.0), 1e-300))}


def assert_bf16_close(g, r, what=""):
    m = metrics(g, r)
    assert m["max_abs"] <= BF16_MAX_ABS and m["mean_rel"] <= BF16_MEAN_REL, (what, m)
    return m


def assert_fp32_close(g, r, what="", tol=FP32_REL):
    m = metrics(g, r)
    assert m["rel"] <= tol, (what, m)
    return m


def bf16_ulp(x):
    """Spacing of the bfloat16 grid at |x| (normal range)."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return np.exp2(e - 7)
