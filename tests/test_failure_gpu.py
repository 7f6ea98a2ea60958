"""Bounded waits: a wait that runs out is reported, and the context stays usable.

The failure is made on purpose, without any fault: through the library's test
hook (mla_debug_absorb_timeout) one epilogue warp of the per-head absorption
kernel withholds a plain software mbarrier arrive, the one that hands the q_C
tile to the W_UK products, and every wait of that kernel is limited to a few
milliseconds.  The MMA issuer's wait then runs out; the kernel records
MLA_ERR_TIMEOUT in the workspace error word, issues no further MMAs, waits for
the loads and MMAs it already issued and exits.  No TMA or MMA completion is
withheld.  The next call, with the hook off, runs normally on the same
workspace and matches the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_45_b200 import _lib as L
from mla_latent_kv_45_b200 import build, synth

from mla_testlib import assert_bf16_close, dev, dev_weights, host, lib_dims, oracle_dims

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    L.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_absorb_wait_timeout_is_reported_and_recovers():
    wl = synth.reduced(synth.V2_BATCH64, "timeout", 60, 3, 0, 0)
    W = synth.make_weights(wl)
    h = synth.make_hidden(wl)
    pos = np.array([5, 700, 4000])
    dims = lib_dims(wl)
    n = L.mla_workspace_size(dims, wl.batch, 5120, 1536, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.mla_workspace_init(ws)
    Wd = dev_weights(W, wl)
    hd = dev(h, wl)
    posd = torch.tensor(pos.astype(np.int32), device="cuda")
    q = torch.zeros(wl.batch, 128, 576, dtype=torch.bfloat16, device="cuda")

    def absorb():
        L.mla_absorb_q(dims, hd, Wd["W_DQ"], Wd["W_UQ"], Wd["W_QR"], Wd["W_UK"], posd, q, ws)

    L.mla_debug_absorb_timeout(True, 5000)   # 5 ms per wait
    try:
        absorb()
        st = L.mla_get_device_error(ws)
    finally:
        L.mla_debug_absorb_timeout(False)
    assert st == 7                            # MLA_ERR_TIMEOUT
    assert L.mla_get_device_error(ws) == 0    # reading clears it

    q.fill_(0)
    absorb()
    assert L.mla_get_device_error(ws) == 0
    ref = oracle.absorb_q(h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], pos, oracle_dims(wl))
    assert_bf16_close(host(q), ref, "q_lat after the timed-out call")
