#!/usr/bin/env python
"""Decode-step benchmark of absorbed MLA over a paged latent cache on B200.

One step = one pass of the whole decode hot path of one layer for a batch:
``mla_cache_append`` (W_DKV + RMSNorm, W_KR + RoPE, paged write) ->
``mla_absorb_q`` (W_DQ, then W_UQ + W_QR + RoPE + W_UK absorption per head) ->
``mla_decode_attn`` (latent attention over every cached row, split-KV merge) ->
``mla_unabsorb_out`` (W_UV, W_O).  The long-context workload (``v2_long``,
131072 rows per sequence) times the attention call alone.

Metric: cached-token x heads per second (sum over sequences of the rows each
new token attends to, times 128 heads, per second), plus the attention call's
fraction of the HBM / bf16 tensor roofline.  Inputs are seeded synthetic data of
the workload's shape; weights N(0, 0.02^2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

The timed region replays the step captured once as a CUDA graph through the
Python API (``DecodeLayer.capture`` -> ``StepGraph.replay``: the same launches
the eager calls make); a second, eager pass records per-call CUDA events for
the breakdown and the attention call's roofline, and a third pass measures the
end-to-end number: pinned host copies of each step's inputs, the replay and
the copy of the output back, all on the device clock.

Multi-GPU: ``--gpus N`` starts N ranks on this node (one per GPU, NCCL),
data-parallel over sequences, each rank its own batch (weak scaling), no
collective on the data path; timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode cached-token·heads/s and % of HBM / bf16 tensor-core roofline"
UNIT = "cached-token·heads/s"
ROW_BYTES = 576 * 2                 # one cached row: c (512) + k_R (64), bf16
INT8_ROW_BYTES = 656                # int8 row: 512 codes, 64 bf16 k_R, scale, padding
FLOP_PER_ROW_HEAD = 2 * 576 + 2 * 512

# Launches of this library per decode step (checked against the ncu launch
# list): append 2 (W_DKV + W_KR projection with its in-cluster split-K sum;
# RMSNorm / RoPE / page write), absorb_q 2 (W_DQ, in-cluster split-K; the fused
# per-head W_UQ + W_QR + RoPE + W_UK kernel), decode_attn 3 (plan, attention,
# merge), unabsorb_out 2 (W_UV; W_O with its in-cluster split-K sum).
LAUNCHES_FULL_STEP = 9
LAUNCHES_ATTENTION = 3


def _find_number(obj, key):
    """The first number stored under ``key`` anywhere in a parsed JSON value."""
    if isinstance(obj, dict):
        v = obj.get(key)
        if isinstance(v, (int, float)) and not isinstance(v, bool):
            return float(v)
        for x in obj.values():
            r = _find_number(x, key)
            if r is not None:
                return r
    elif isinstance(obj, list):
        for x in obj:
            r = _find_number(x, key)
            if r is not None:
                return r
    return None


def peaks(path=None):
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source): the measured
    peaks of this machine's B200s when MEASURED_PEAKS.json holds them (at any depth),
    else the pool's earlier measurement."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
            hbm, tf = _find_number(d, "hbm_gbs"), _find_number(d, "bf16_tflops")
            if hbm and tf:
                return hbm, tf, _find_number(d, "bf16_tflops_sustained"), "measured"
        except (OSError, ValueError):
            pass
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

def workload(name, rank):
    from mla_latent_kv_45_b200 import synth
    base = synth.WORKLOADS[name]
    # each rank holds its own shard of sequences (distinct seeds), same shape
    return dataclasses.replace(base, wid=base.wid + 100 * rank)


def attention_only(wl) -> bool:
    return wl.new_tokens == 0


def prefill(wl) -> bool:
    """A chunk of new tokens per sequence: run as one entry per token sharing the
    sequence's page-table row, entry t attending to rows 0 .. p0 + t."""
    return wl.new_tokens > 1


def describe(wl):
    if attention_only(wl):
        what = "latent attention only (plan + attention + split merge) over the cached rows"
        rows = f"{wl.prior_min} rows per sequence (the query's own included)"
    elif prefill(wl):
        what = ("chunked prefill through the decode calls: the chunk's tokens as entries "
                "sharing the page table row (causal), append + absorb_q + attention + unabsorb")
        rows = f"{wl.prior_min} cached rows + a {wl.new_tokens}-token chunk"
    else:
        what = "full layer step: append + absorb_q (W_DQ) + attention + unabsorb (W_UV, W_O)"
        rows = f"cached rows {wl.prior_min}..{wl.prior_max} + {wl.new_tokens} new"
    fmt = ("; int8 cache rows (codes x 2^e per row, k_R bf16, 656 B)" if wl.cache == "int8"
           else "")
    return (f"{wl.name}: batch {wl.batch}/GPU, {wl.n_heads} heads, d_model {wl.d_model}, "
            f"q_lora {wl.d_q}, d_c {wl.d_c}, d_rope {wl.d_rope}, d_nope {wl.d_nope}, d_v {wl.d_v}, "
            f"{rows}, {wl.page_size}-row pages{' (shuffled)' if wl.shuffle_pages else ''}{fmt}; "
            f"{what}")


def row_bytes(wl):
    return INT8_ROW_BYTES if wl.cache == "int8" else ROW_BYTES


def attended_lengths(wl, prior):
    """Rows each query attends to (per token of a prefill chunk)."""
    if attention_only(wl):
        return prior
    if prefill(wl):
        return np.concatenate([p + 1 + np.arange(wl.new_tokens) for p in prior])
    return prior + 1


def algorithmic(wl, lens):
    """Bytes / FLOPs that any implementation must move / do, per step and per attention call."""
    B, H = len(lens), wl.n_heads      # queries (a prefill chunk's tokens count one each)
    rows = int(lens.sum())
    if prefill(wl):
        # each cached row is needed once per chunk, not once per query
        cached = int(wl.batch * (wl.prior_max + wl.new_tokens))
        attn_bytes = cached * row_bytes(wl) + B * H * 576 * 2 + B * H * 512 * 2
    else:
        attn_bytes = rows * row_bytes(wl) + B * H * 576 * 2 + B * H * 512 * 2  # cache + q_lat + z
    attn_flops = rows * H * FLOP_PER_ROW_HEAD
    if attention_only(wl):
        return dict(rows=rows, attn_bytes=attn_bytes, attn_flops=attn_flops,
                    step_bytes=attn_bytes, step_flops=attn_flops, params=0)
    dq = wl.d_q or wl.d_model
    params = (wl.d_c + wl.d_rope) * wl.d_model + (wl.d_q * wl.d_model if wl.d_q else 0) \
        + H * (wl.d_nope + wl.d_rope) * dq + H * wl.d_nope * wl.d_c + H * wl.d_v * wl.d_c \
        + wl.d_model * H * wl.d_v
    step_bytes = attn_bytes + 2 * params + B * row_bytes(wl) + 2 * B * wl.d_model * 2
    step_flops = attn_flops + 2 * B * params
    return dict(rows=rows, attn_bytes=attn_bytes, attn_flops=attn_flops, step_bytes=step_bytes,
                step_flops=step_flops, params=params)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (read-only NVML queries)
# ---------------------------------------------------------------------------

class ClockSampler:
    """Polls the SM clock, the power draw and the active clock-event reasons of
    one GPU through NVML every ~0.5 ms on a background thread, so that even a
    timed region of a few milliseconds holds samples.  Reads only."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("sw_power_cap", 0x4))

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def _poll(self):
        import pynvml
        while not self._stop.is_set():
            try:
                t = time.time()
                sm = pynvml.nvmlDeviceGetClockInfo(self._h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                pw = pynvml.nvmlDeviceGetPowerUsage(self._h) / 1000.0
            except Exception:
                return
            self.samples.append((t, sm, rs, pw))
            time.sleep(0.0005)

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, windows):
        """Samples inside the given (t0, t1) wall-clock windows."""
        if self._thread is None or not self.samples:
            return None
        inside = [s for s in self.samples if any(t0 <= s[0] <= t1 for t0, t1 in windows)]
        used = inside or self.samples
        reasons = sorted({name for s in used for name, bit in self.REASONS if s[2] & bit})
        return {"sm_mhz": statistics.median(s[1] for s in used), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "power_w_median": statistics.median(s[3] for s in used),
                "samples_in_timed_region": len(inside), "source": "nvml, ~0.5 ms polling"}


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(nproc, argv):
    """Re-runs this script under torch.distributed.run with one rank per GPU
    (used when --gpus N > 1 is given outside a torchrun launch)."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def setup_dist(args, backend="nccl"):
    """Process group from the torchrun environment (one rank per GPU; ``gloo`` for
    host-only checks).  Sequences are sharded by rank; the data path has no collective."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return rank, world, local


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings (the job takes as long as its slowest rank)."""
    import torch
    t = torch.tensor(values, device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------------------
# the oracle's CPU time (baseline only; never on the timed path)
# ---------------------------------------------------------------------------

def _threads():
    try:
        import threadpoolctl
        return max((p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        return 1


def _oracle_dims(wl):
    import oracle
    return oracle.Dims(n_heads=wl.n_heads, d_c=wl.d_c, d_rope=wl.d_rope, d_nope=wl.d_nope,
                       d_v=wl.d_v, rope_base=wl.rope_base, rms_eps=wl.rms_eps,
                       rope_layout=wl.rope_layout)


def _oracle_unit(wl, W, pc, h, q):
    """f(b, n): the oracle's work for sequence b over its first n attended rows
    (a whole un-absorbed decode step, or the latent attention alone); int8 rows
    are read back through the oracle's dequantisation."""
    import oracle
    od = _oracle_dims(wl)

    def rows(b, n):
        if wl.cache != "int8":
            return pc.rows_f32(b, n)
        codes, exps, k_r = pc.fields(b, n)
        return np.concatenate([oracle.dequantize_int8_pow2(codes, exps), k_r], axis=1)

    if attention_only(wl):
        return lambda b, n: oracle.attend_latent(q[b], rows(b, n), od)
    return lambda b, n: oracle.decode_step(h[b:b + 1], [rows(b, n - 1)], W, od)


def cpu_baseline_sample(wl, W, pc, h, q, lens, budget_s=20.0):
    """The oracle on a bounded sample of the workload: one sequence over a prefix."""
    f = _oracle_unit(wl, W, pc, h, q)
    t = time.perf_counter()
    f(0, 64)
    per_row = (time.perf_counter() - t) / 64
    n = int(min(lens[0], max(64, budget_s / max(per_row, 1e-9))))
    t = time.perf_counter()
    f(0, n)
    dt = time.perf_counter() - t
    form = ("latent attention" if attention_only(wl) else "whole un-absorbed decode step")
    return {"value": n * wl.n_heads / dt, "unit": UNIT, "cores": int(_threads()), "kind": "oracle",
            "sample": f"sequence 0 of {wl.name}, first {n} attended rows (new token included), "
                      f"all {wl.n_heads} heads, one fp64 {form} ({dt:.1f} s)",
            "host_cpus": os.cpu_count()}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def run_mine(args):
    import torch
    from mla_latent_kv_45_b200 import _lib as L
    from mla_latent_kv_45_b200 import build, synth
    from mla_latent_kv_45_b200.layer import DecodeLayer, StepGraph

    rank, world, local = setup_dist(args)
    torch.cuda.set_device(local)
    build.build()
    wl = workload(args.workload, rank)
    attn_only = attention_only(wl)
    prior = synth.make_prior_lengths(wl)
    lens = attended_lengths(wl, prior)
    int8 = wl.cache == "int8"
    pc = synth.make_paged_cache_int8(wl, prior) if int8 else synth.make_paged_cache(wl, prior)
    W = None if attn_only else synth.make_weights(wl)
    h = None if attn_only else synth.make_hidden(wl)
    q = synth.make_q_lat(wl) if attn_only else None
    dims = L.Dims(wl.n_heads, wl.d_c, wl.d_rope, wl.d_nope, wl.d_v, wl.page_size, L.MLA_BF16,
                  wl.rope_layout, wl.rope_base, wl.rms_eps,
                  cache_format=L.MLA_CACHE_INT8 if int8 else L.MLA_CACHE_NATIVE)
    dev = torch.device("cuda", local)
    bf = lambda a: torch.from_numpy(a).to(dev).to(torch.bfloat16)
    if int8:
        pool = torch.from_numpy(pc.pool).to(dev)
    else:
        pool = torch.from_numpy(pc.pool.view(np.int16)).to(dev).view(torch.bfloat16)
    cache = L.PagedCache(pool, torch.from_numpy(pc.block_table).to(dev),
                         torch.from_numpy(lens.astype(np.int32)).to(dev))
    stream = torch.cuda.current_stream()
    if attn_only:
        # attention alone: q_lat in, z / lse out
        q_dev = bf(q)
        n_ws = L.mla_workspace_size(dims, wl.batch, 64, 0, args.num_splits)
        ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
        L.mla_workspace_init(ws)
        z = torch.empty(wl.batch, wl.n_heads, wl.d_c, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(wl.batch, wl.n_heads, dtype=torch.float32, device=dev)

        def step(e=None, st=None):
            st = st or stream
            if e:
                e[4].record(st)
            L.mla_decode_attn(dims, cache, q_dev, z, lse, args.num_splits, ws, st)
            if e:
                e[5].record(st)

        def device_error():
            return L.mla_get_device_error(ws)

        def capture():
            step()
            torch.cuda.synchronize()
            return StepGraph(lambda st: step(st=st), z)

        def second_set():
            # its own input, output and workspace buffers over the same cache
            q2, z2, l2 = q_dev.clone(), torch.empty_like(z), torch.empty_like(lse)
            ws2 = torch.empty_like(ws)
            L.mla_workspace_init(ws2)

            def run(st):
                L.mla_decode_attn(dims, cache, q2, z2, l2, args.num_splits, ws2, st)

            run(stream)
            torch.cuda.synchronize()
            return StepGraph(run, z2), [q2], z2, lambda: L.mla_get_device_error(ws2)

        inputs, output = [q_dev], z
        launches = LAUNCHES_ATTENTION
    else:
        Wd = {k: (None if v is None else bf(v)) for k, v in W.items()}
        if prefill(wl):
            # one entry per chunk token, all sharing their sequence's page-table row
            T = wl.new_tokens
            hd = bf(synth.make_hidden(wl, n=wl.batch * T))
            pos = torch.from_numpy(np.concatenate([p + np.arange(T) for p in prior])
                                   .astype(np.int32)).to(dev)
            cache = L.PagedCache(pool, torch.from_numpy(np.repeat(pc.block_table, T, axis=0))
                                 .to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev))
        else:
            hd = bf(h)
            pos = torch.from_numpy(prior.astype(np.int32)).to(dev)
        layer = DecodeLayer(dims, Wd, len(lens), args.num_splits, device=dev)

        def step(e=None):
            layer.step(cache, hd, pos, stream, e)

        def capture():
            return layer.capture(cache, hd, pos)

        def second_set():
            # another layer object (workspaces, outputs) over the same weights and
            # pool, with its own input buffers and sequence lengths
            layer2 = DecodeLayer(dims, Wd, len(lens), args.num_splits, device=dev)
            h2, p2 = hd.clone(), pos.clone()
            cache2 = L.PagedCache(cache.pool, cache.block_table, cache.seq_lens.clone())
            return (layer2.capture(cache2, h2, p2), [h2, p2, cache2.seq_lens], layer2.out,
                    layer2.device_error)

        device_error = layer.device_error
        inputs, output = [hd, pos, cache.seq_lens], layer.out
        launches = LAUNCHES_FULL_STEP

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = device_error()
    if st != 0:
        raise RuntimeError(f"device error {L.STATUS.get(st)} during warm-up")

    # one step captured as a CUDA graph through the Python API (the same
    # launches, replayed with no per-kernel host work)
    graph = capture()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}") if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.2)
    windows = []

    # ---- timed region: K steps, barrier + synchronize on both sides
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    windows.append((t_wall0, time.time()))
    if world > 1:
        torch.distributed.barrier()
    elapsed = start.elapsed_time(end)  # ms
    st = device_error()
    if st != 0:
        raise RuntimeError(f"device error {L.STATUS.get(st)} in the timed region")

    # ---- per-call breakdown (eager, events around each call on its own stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    t_b0 = time.time()
    for k in range(args.steps):
        step(ev[k])
    torch.cuda.synchronize()
    windows.append((t_b0, time.time()))
    if attn_only:
        per_call = np.array([[0.0, 0.0, e[4].elapsed_time(e[5]), 0.0] for e in ev])
    else:
        per_call = np.array([[e[0].elapsed_time(e[1]), e[2].elapsed_time(e[3]),
                              e[4].elapsed_time(e[5]), e[5].elapsed_time(e[6])] for e in ev])

    # ---- end-to-end through the Python API with host buffers, as a serving loop
    # runs it: two buffer sets, each with its step captured (DecodeLayer.capture);
    # step k copies its inputs from pinned host memory into set k % 2 on a copy
    # stream, replays set k % 2's step, and copies its output back to pinned host
    # memory on a third stream, so the copies of steps k + 1 and k - 1 overlap the
    # compute of step k.  Every step's copies are inside the timed region.
    graph2, inputs2, output2, device_error2 = second_set()
    sets = [(graph, inputs, output), (graph2, inputs2, output2)]
    host_in = [t.cpu().pin_memory() for t in inputs]
    out_host = [torch.empty(output.shape, dtype=output.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for i in range(2):
        ev_done[i].record(stream)
        ev_out[i].record(stream)

    def e2e_step(k):
        g, ins, out = sets[k % 2]
        i = k % 2
        s_in.wait_event(ev_done[i])          # step k - 2 has read this set's inputs
        with torch.cuda.stream(s_in):
            for d, hbuf in zip(ins, host_in):
                d.copy_(hbuf, non_blocking=True)
        ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        stream.wait_event(ev_out[i])         # step k - 2's output has been copied out
        g.replay()
        ev_done[i].record(stream)
        s_out.wait_event(ev_done[i])
        with torch.cuda.stream(s_out):
            out_host[i].copy_(out, non_blocking=True)
        ev_out[i].record(s_out)

    for k in range(4):
        e2e_step(k)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(args.steps):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if clocks:
        clocks.stop()
    for err in (device_error(), device_error2()):
        if err != 0:
            raise RuntimeError(f"device error {L.STATUS.get(err)} in the end-to-end pass")

    elapsed, e2e_ms, attn_ms_total = max_over_ranks([elapsed, e2e_ms, per_call[:, 2].sum()],
                                                    world, dev)

    alg = algorithmic(wl, lens)
    hbm, tf, tf_sus, src = peaks()
    ms_step = elapsed / args.steps
    value = alg["rows"] * wl.n_heads * world / (ms_step / 1e3)
    # the attention call's time: the timed step itself when the step is the
    # call; otherwise the eager pass's events around the call
    attn_ms = ms_step if attn_only else attn_ms_total / args.steps
    t_bytes = alg["attn_bytes"] / (hbm * 1e9)
    t_flops = alg["attn_flops"] / (tf * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    if bound == "hbm":
        achieved, peak, unit = alg["attn_bytes"] / (attn_ms / 1e3) / 1e9, hbm, "GB/s"
    else:
        achieved, peak, unit = alg["attn_flops"] / (attn_ms / 1e3) / 1e12, tf, "TFLOP/s"
    step_t = max(alg["step_bytes"] / (hbm * 1e9), alg["step_flops"] / (tf * 1e12))
    h2d = sum(t.numel() * t.element_size() for t in inputs)
    d2h = output.numel() * output.element_size()
    l2 = ("no flush: per-step inputs (cache %.0f MB%s) exceed the 126 MB L2"
          % (alg["rows"] * row_bytes(wl) / 1e6,
             "" if attn_only else " + weights %.0f MB" % (2 * alg["params"] / 1e6)))
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(wl), "batch_per_gpu": wl.batch,
                   "global_batch": wl.batch * world, "cached_rows_per_step": alg["rows"],
                   "parallelism": f"dp{world} (sequences sharded, no collective)",
                   "l2": l2, "num_splits": args.num_splits,
                   "timed": "the step captured once (DecodeLayer.capture), replayed K times"},
        "roofline": {"kernel": "mla_decode_attn (plan + attention + split merge)",
                     "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "traffic": stored_traffic(wl.name),
                     "peak_source": src,
                     "algorithmic_bytes": alg["attn_bytes"], "algorithmic_flops": alg["attn_flops"],
                     "ms_per_launch": attn_ms,
                     "timing": ("the timed step (the step is the call)" if attn_only else
                                "CUDA events around each call in an eager pass of K steps")},
        "step_roofline": {"bytes": alg["step_bytes"], "flops": alg["step_flops"],
                          "roofline_ms": step_t * 1e3, "frac": step_t * 1e3 / ms_step},
        "breakdown_ms": dict(zip(["cache_append", "absorb_q", "decode_attn", "unabsorb_out"],
                                 [float(x) for x in per_call.mean(0)])),
        "e2e": {"value": alg["rows"] * wl.n_heads * world / (e2e_ms / args.steps / 1e3),
                "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms / args.steps,
                "how": "per step: pinned host copies of the inputs into one of two buffer "
                       "sets (copy stream), StepGraph.replay() of that set's captured step, "
                       "pinned copy of the output back (third stream); copies of neighbouring "
                       "steps overlap the compute"},
        "gpu_launches": launches * args.steps,
    }
    if rank == 0:
        res["clocks"] = clocks.summary(windows) if clocks else None
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_sample(wl, W, pc, h, q, lens)
        print(json.dumps(res), flush=True)
    del graph, graph2, sets
    if world > 1:
        torch.distributed.destroy_process_group()


ATTN_SOURCES = ("attn_sm100.cu", "kernels_simt.cu", "ptx.cuh", "common.cuh", "kernels.h", "sm100.h")


def stored_traffic(workload, tfile=None):
    """DRAM bytes per decode-attention call from the committed ncu capture, or
    None when the capture is for another workload or for other kernel sources."""
    tfile = tfile or os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(tfile):
        return None
    with open(tfile) as f:
        tinfo = json.load(f)
    if tinfo.get("workload") != workload or tinfo.get("kernel_rev") != kernel_revision():
        return None
    return tinfo.get("dram_bytes_per_launch")


def kernel_revision():
    """Hash of the sources of the decode-attention call's kernels (plan, attention,
    merge): a stored ncu traffic figure is only valid for them."""
    import hashlib
    hsh = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "mla_latent_kv_45_b200", "csrc", name), "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()[:16]


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mla_latent_kv_45_b200 import synth
    wl = workload(args.workload, 0)
    prior = synth.make_prior_lengths(wl)
    lens = attended_lengths(wl, prior)
    pc = (synth.make_paged_cache_int8(wl, prior) if wl.cache == "int8"
          else synth.make_paged_cache(wl, prior))
    attn_only = attention_only(wl)
    W = None if attn_only else synth.make_weights(wl)
    h = None if attn_only else synth.make_hidden(wl)
    q = synth.make_q_lat(wl) if attn_only else None
    f = _oracle_unit(wl, W, pc, h, q)
    # size each step's sample so the whole run stays within ~2 minutes
    t = time.perf_counter()
    f(0, 64)
    per_row = (time.perf_counter() - t) / 64
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(lens.min(), max(16, budget / max(per_row, 1e-9))))

    for k in range(args.warmup):
        f(k % wl.batch, n)
    t0 = time.perf_counter()
    for k in range(args.steps):
        f(k % wl.batch, n)
    dt = time.perf_counter() - t0
    value = n * wl.n_heads * args.steps / dt
    form = "latent attention" if attn_only else "whole un-absorbed fp64 decode step"
    sample = (f"each step: one sequence of {wl.name} (cycling over its {wl.batch}), first {n} "
              f"attended rows incl. the new token, all {wl.n_heads} heads, {form}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": describe(wl)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(_threads()), "kind": "oracle",
                         "sample": sample, "host_cpus": os.cpu_count()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------
# multi-rank plumbing check without a GPU
# ---------------------------------------------------------------------------

def run_rank_check(args):
    """Each rank reports a rank-dependent timing through the same max-over-ranks
    reduction the bench uses (gloo, no GPU); rank 0 prints one line."""
    rank, world, _ = setup_dist(args, backend="gloo")
    wl = workload(args.workload, rank)
    got = max_over_ranks([1.0 + rank, float(wl.wid)], world, "cpu")
    if rank == 0:
        print(json.dumps({"n_gpus": world, "max_ms": got[0], "max_wid": got[1]}), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", default="v2_batch64")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rank-check", action="store_true",
                    help="run only the multi-rank plumbing on CPU (gloo), no GPU work")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    if args.rank_check:
        run_rank_check(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_mine(args)


if __name__ == "__main__":
    main()
