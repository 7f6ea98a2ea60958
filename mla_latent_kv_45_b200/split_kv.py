"""Decode attention over sequences whose cached rows are spread across devices.

A very long sequence need not fit, or be read, on one GPU: each rank holds a
contiguous range of every sequence's pages (its share), attends over its share
alone, and the ranks then exchange the partial softmaxes and merge them.  The
partial of a share is (O, m, l) with m the largest logit, l the sum of
e^(logit - m) and O the e^(logit - m)-weighted sum of the latent rows
(``mla_decode_attn_partial``); z = sum_j e^(m_j - M) O_j / sum_j e^(m_j - M) l_j
over the shares (``mla_merge_partials``), which is the same softmax taken in
pieces.  The exchange is one all-gather per call of O [B, H, d_c] fp32 and
m, l [B, H]: about 257 KB per sequence per rank at the DeepSeek-V2 sizes,
small next to the rows each rank reads.

``shard_pages`` is host-side bookkeeping (which pages and rows each rank
holds); ``CrossDeviceAttention`` runs the partial, the all-gather
(``torch.distributed``, NCCL on GPUs) and the merge.  Every arithmetic step
runs in the CUDA library.
"""

from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np
import torch

from . import _lib as L


def shard_pages(block_table: np.ndarray, seq_lens: Sequence[int], page_size: int,
                world: int) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Splits each sequence's pages into ``world`` contiguous ranges.

    Returns, per rank r, ``(block_table_r, seq_lens_r)``: the rank's pages of
    each sequence in logical order (padded with -1) and the number of rows they
    hold.  Rank r takes pages [r n / world, (r + 1) n / world) of a sequence
    with n pages; a rank whose range is empty holds 0 rows.
    """
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens, dtype=np.int64)
    B = bt.shape[0]
    n_pages = (lens + page_size - 1) // page_size
    out = []
    for r in range(world):
        lo = n_pages * r // world
        hi = n_pages * (r + 1) // world
        width = max(int((hi - lo).max(initial=0)), 1)
        bt_r = np.full((B, width), -1, dtype=np.int32)
        rows = np.zeros(B, dtype=np.int32)
        for b in range(B):
            k = int(hi[b] - lo[b])
            bt_r[b, :k] = bt[b, lo[b]:hi[b]]
            rows[b] = max(0, min(int(lens[b]), int(hi[b]) * page_size) - int(lo[b]) * page_size)
        out.append((bt_r, rows))
    return out


def gather_partials(O: torch.Tensor, m: torch.Tensor, l: torch.Tensor, group=None):
    """All-gather of every rank's partial: stacks [world, ...] in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    outs = []
    for t in (O, m, l):
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        outs.append(torch.stack(parts))
    return outs


class CrossDeviceAttention:
    """Decode attention of a batch whose rows are sharded across the ranks of a
    process group (one rank per GPU).  Every rank passes its own share of the
    cache and the full q_lat, and receives the full z / lse."""

    def __init__(self, dims: L.Dims, batch: int, group=None, num_splits: int = 0, device="cuda"):
        self.dims, self.batch, self.group, self.num_splits = dims, batch, group, num_splits
        H, d_c = dims.n_heads, dims.d_c
        nbytes = L.mla_workspace_size(dims, batch, 64, 0, num_splits)
        if nbytes == 0:
            raise ValueError("unsupported dims for the workspace")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        L.mla_workspace_init(self.ws)
        self.O = torch.empty(batch, H, d_c, dtype=torch.float32, device=device)
        self.m = torch.empty(batch, H, dtype=torch.float32, device=device)
        self.l = torch.empty(batch, H, dtype=torch.float32, device=device)

    def __call__(self, local_cache: L.PagedCache, q_lat: torch.Tensor, z: torch.Tensor,
                 lse: torch.Tensor = None, stream=None):
        L.mla_decode_attn_partial(self.dims, local_cache, q_lat, self.O, self.m, self.l,
                                  self.num_splits, self.ws, stream)
        gO, gm, gl = gather_partials(self.O, self.m, self.l, self.group)
        L.mla_merge_partials(self.dims, gO, gm, gl, z, lse, stream)
        return z

    def device_error(self) -> int:
        return L.mla_get_device_error(self.ws)
