"""Cross-device split-KV on CPU: page sharding and the partial exchange.

Two ``gloo`` ranks each take their share of every sequence's pages
(``split_kv.shard_pages``), compute the partial softmax of that share with the
fp64 oracle, exchange the partials with the same ``gather_partials`` the GPU
path uses, and merge them with the oracle's split combine; the result must be
the unsplit attention over all rows.  The CUDA partial and merge kernels are
checked on one GPU in ``test_split_kv_gpu.py``.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

LENS = [1, 64, 65, 300, 1000]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from mla_latent_kv_45_b200 import synth
    wl = synth.reduced(synth.TINY, "split_kv_cpu", 70, len(LENS), 0, 0, new_tokens=0,
                       page_size=16)
    pc = synth.make_paged_cache(wl, np.array(LENS))
    return wl, pc, synth.make_q_lat(wl)


def partial_of(q, rows, od):
    import oracle
    if len(rows) == 0:
        return np.zeros((q.shape[0], od.d_c)), np.full(q.shape[0], -np.inf), np.zeros(q.shape[0])
    return oracle.split_partial(q, rows, od)


def test_shards_cover_every_row_once():
    from mla_latent_kv_45_b200.split_kv import shard_pages
    wl, pc, _ = _case()
    for world in (1, 2, 3, 8):
        shards = shard_pages(pc.block_table, LENS, wl.page_size, world)
        for b, Lb in enumerate(LENS):
            rows = []
            for bt_r, lens_r in shards:
                n = int(lens_r[b])
                idx = np.arange(n)
                rows.append(pc.pool[bt_r[b][idx // wl.page_size], idx % wl.page_size])
            np.testing.assert_array_equal(np.concatenate(rows), pc.rows_f32(b, Lb))
        # a one-page sequence leaves the other shares empty
        assert sum(int(l_r[0] > 0) for _, l_r in shards) == 1


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import oracle
    from mla_latent_kv_45_b200.split_kv import gather_partials, shard_pages
    dist.init_process_group("gloo")
    wl, pc, q = _case()
    od = oracle.Dims(n_heads=wl.n_heads, d_c=wl.d_c, d_rope=wl.d_rope, d_nope=wl.d_nope,
                     d_v=wl.d_v)
    bt_r, lens_r = shard_pages(pc.block_table, LENS, wl.page_size, world)[rank]
    O, m, l = [], [], []
    for b in range(len(LENS)):
        idx = np.arange(int(lens_r[b]))
        rows = pc.pool[bt_r[b][idx // wl.page_size], idx % wl.page_size]
        o_b, m_b, l_b = partial_of(q[b], rows, od)
        O.append(o_b), m.append(m_b), l.append(l_b)
    gO, gm, gl = gather_partials(torch.from_numpy(np.stack(O)), torch.from_numpy(np.stack(m)),
                                 torch.from_numpy(np.stack(l)))
    errs = []
    for b, Lb in enumerate(LENS):
        z, lse = oracle.combine_splits(gO[:, b].numpy(), gm[:, b].numpy(), gl[:, b].numpy())
        zr, lr = oracle.attend_latent(q[b], pc.rows_f32(b, Lb), od)
        errs.append(max(np.abs(z - zr).max(), np.abs(lse - lr).max()))
    out.put((rank, max(errs)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_exchange_and_merge():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [r for r, _ in res] == [0, 1]
    assert all(err < 1e-12 for _, err in res), res
