"""One decode step of an MLA layer through the four C-ABI calls.

The order is the pages' per-token inference flow ("解耦 RoPE（MLA 下）" §五):
append the new token's [c ; k_R] row, build the absorbed query, attend over
the whole cache (the new row included), then up-project.  Device tensors only;
every step runs in the CUDA library.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _lib as L


class DecodeLayer:
    """Weights of one layer (device tensors, ``[out, in]`` layout) plus a workspace."""

    def __init__(self, dims: L.Dims, weights: dict, batch: int, num_splits: int = 0,
                 device="cuda"):
        self.dims = dims
        self.w = weights
        self.batch = batch
        self.num_splits = num_splits
        self.d_model = weights["W_DKV"].shape[1]
        self.d_q = weights["W_DQ"].shape[0] if weights.get("W_DQ") is not None else 0
        nbytes = L.mla_workspace_size(dims, batch, self.d_model, self.d_q, num_splits)
        if nbytes == 0:
            raise ValueError("unsupported dims for the workspace")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        L.mla_workspace_init(self.ws)
        # the cache append runs on a second stream, beside the query absorption
        # (the two only meet at the attention), with a workspace of its own
        self.ws_append = torch.empty(nbytes, dtype=torch.uint8, device=device)
        L.mla_workspace_init(self.ws_append)
        self.side = torch.cuda.Stream(device=device)
        H, dt = dims.n_heads, dims.torch_dtype
        self.q_lat = torch.empty(batch, H, dims.d_c + dims.d_rope, dtype=dt, device=device)
        self.z = torch.empty(batch, H, dims.d_c, dtype=dt, device=device)
        self.lse = torch.empty(batch, H, dtype=torch.float32, device=device)
        d_out = self.d_model if weights.get("W_O") is not None else H * dims.d_v
        self.out = torch.empty(batch, d_out, dtype=dt, device=device)

    def step(self, cache: L.PagedCache, h: torch.Tensor, positions: torch.Tensor,
             stream=None, events=None) -> torch.Tensor:
        """Appends h's rows at ``positions`` and returns the layer output.

        ``cache.seq_lens`` must already count the new rows (positions + 1).
        The append runs on a side stream concurrently with the query absorption;
        the attention waits for both.  ``events`` (7 CUDA events, optional) are
        recorded around each call: append [0, 1] on the side stream, absorb
        [2, 3], attention [4, 5] and un-absorption [5, 6] on the main stream.
        """
        w, d = self.w, self.dims
        main = stream if stream is not None else torch.cuda.current_stream()
        side = self.side
        side.wait_stream(main)
        if events:
            events[0].record(side)
        L.mla_cache_append(d, cache, h, w["W_DKV"], w["W_KR"], w["gamma"], positions,
                           self.ws_append, side)
        if events:
            events[1].record(side)
            events[2].record(main)
        L.mla_absorb_q(d, h, w.get("W_DQ"), w["W_UQ"], w["W_QR"], w["W_UK"], positions,
                       self.q_lat, self.ws, main)
        if events:
            events[3].record(main)
        main.wait_stream(side)
        if events:
            events[4].record(main)
        L.mla_decode_attn(d, cache, self.q_lat, self.z, self.lse, self.num_splits, self.ws, main)
        if events:
            events[5].record(main)
        L.mla_unabsorb_out(d, self.z, w["W_UV"], w.get("W_O"), self.out, self.ws, main)
        if events:
            events[6].record(main)
        return self.out

    def capture(self, cache: L.PagedCache, h: torch.Tensor, positions: torch.Tensor
                ) -> "StepGraph":
        """The decode step over these buffers, captured once as a CUDA graph.

        The graph reads ``h``, ``positions``, ``cache.seq_lens`` and the cache
        in place and writes ``self.out`` (and the cache row): copy each step's
        inputs into those buffers and call ``replay()``.  One eager step runs
        first so that every one-time set-up (per-device kernel attributes)
        happens outside the capture.
        """
        self.step(cache, h, positions)
        torch.cuda.synchronize()
        return StepGraph(lambda s: self.step(cache, h, positions, s), self.out)

    def device_error(self) -> int:
        """Synchronises; returns the first nonzero device status of both workspaces."""
        st = L.mla_get_device_error(self.ws_append, self.side)
        st2 = L.mla_get_device_error(self.ws)
        return st if st != 0 else st2


class StepGraph:
    """A CUDA graph of one call sequence issued by ``fn(stream)``; ``replay``
    launches the same kernels on the current stream with no per-kernel host
    work."""

    def __init__(self, fn, out: torch.Tensor):
        self.out = out
        self.graph = torch.cuda.CUDAGraph()
        main = torch.cuda.current_stream()
        cap = torch.cuda.Stream(device=main.device)
        cap.wait_stream(main)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(self.graph, stream=cap):
                fn(cap)
        main.wait_stream(cap)

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.out
