#!/usr/bin/env python
"""Decode-step benchmark of absorbed MLA over a paged latent cache on B200.

One step = one pass of the whole decode hot path of one layer for a batch:
``mla_cache_append`` (W_DKV + RMSNorm, W_KR + RoPE, paged write) ->
``mla_absorb_q`` (W_DQ, W_UQ, W_QR + RoPE, W_UK absorption) ->
``mla_decode_attn`` (latent attention over every cached row, split-KV merge) ->
``mla_unabsorb_out`` (W_UV, W_O).

Metric: cached-token x heads per second (sum over sequences of the rows each
new token attends to, times 128 heads, per second), plus the attention call's
fraction of the HBM / bf16 tensor roofline.  Inputs are seeded synthetic data of
the workload's shape; weights N(0, 0.02^2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU (torchrun): data-parallel over sequences, each rank its own batch
(weak scaling), no collective on the data path; timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
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
FLOP_PER_ROW_HEAD = 2 * 576 + 2 * 512


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

def workload(name, rank):
    from mla_latent_kv_45_b200 import synth
    base = synth.WORKLOADS[name]
    # each rank holds its own shard of sequences (distinct seeds), same shape
    return dataclasses.replace(base, wid=base.wid + 100 * rank)


def describe(wl, lens):
    return (f"{wl.name}: batch {wl.batch}/GPU, {wl.n_heads} heads, d_model {wl.d_model}, "
            f"q_lora {wl.d_q}, d_c {wl.d_c}, d_rope {wl.d_rope}, d_nope {wl.d_nope}, d_v {wl.d_v}, "
            f"cached rows {wl.prior_min}..{wl.prior_max} + {wl.new_tokens} new, "
            f"{wl.page_size}-row pages{' (shuffled)' if wl.shuffle_pages else ''}; "
            f"full layer step: append + absorb_q (W_DQ) + attention + unabsorb (W_UV, W_O)")


def algorithmic(wl, lens):
    """Bytes / FLOPs that any implementation must move / do, per step and per attention call."""
    B, H = wl.batch, wl.n_heads
    rows = int(lens.sum())
    attn_bytes = rows * ROW_BYTES + B * H * 576 * 2 + B * H * 512 * 2   # cache + q_lat + z
    attn_flops = rows * H * FLOP_PER_ROW_HEAD
    dq = wl.d_q or wl.d_model
    params = (wl.d_c + wl.d_rope) * wl.d_model + (wl.d_q * wl.d_model if wl.d_q else 0) \
        + H * (wl.d_nope + wl.d_rope) * dq + H * wl.d_nope * wl.d_c + H * wl.d_v * wl.d_c \
        + wl.d_model * H * wl.d_v
    step_bytes = attn_bytes + 2 * params + B * ROW_BYTES + 2 * B * wl.d_model * 2
    step_flops = attn_flops + 2 * B * params
    return dict(rows=rows, attn_bytes=attn_bytes, attn_flops=attn_flops, step_bytes=step_bytes,
                step_flops=step_flops, params=params)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(self.gpu_id)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        if self.proc is None:
            return None
        inside = [s for t, s in self.samples if t0 <= t <= t1]
        # a short timed region may hold no sample: then use the ones within 0.25 s of it
        near = [s for t, s in self.samples if t0 - 0.25 <= t <= t1 + 0.25]
        used = inside or near or [s for _, s in self.samples]
        sm, mx, reasons = [], [], set()
        for s in used:
            try:
                sm.append(float(s[1]))
                mx.append(float(s[2]))
            except (ValueError, IndexError):
                continue
            for name, v in zip(self.NAMES, s[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(used), "samples_in_timed_region": len(inside),
                "sample_interval_ms": 20}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

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


def cpu_baseline_sample(wl, W, pc, h, lens, budget_s=20.0):
    """The oracle's whole decode step (un-absorbed form) on a bounded sample."""
    import oracle
    od = oracle.Dims(n_heads=wl.n_heads, d_c=wl.d_c, d_rope=wl.d_rope, d_nope=wl.d_nope,
                     d_v=wl.d_v, rope_base=wl.rope_base, rms_eps=wl.rms_eps,
                     rope_layout=wl.rope_layout)
    # calibrate on a short prefix of sequence 0, then size the sample to the budget
    t = time.perf_counter()
    oracle.decode_step(h[:1], [pc.rows_f32(0, 63)], W, od)
    per_row = (time.perf_counter() - t) / 64
    n = int(min(lens[0], max(64, budget_s / max(per_row, 1e-9))))
    t = time.perf_counter()
    oracle.decode_step(h[:1], [pc.rows_f32(0, n - 1)], W, od)
    dt = time.perf_counter() - t
    try:
        import threadpoolctl
        threads = max((p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        threads = 1
    return {"value": n * wl.n_heads / dt, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": f"sequence 0 of {wl.name}, first {n} cached rows (new token included), "
                      f"all {wl.n_heads} heads, one whole un-absorbed fp64 decode step "
                      f"({dt:.1f} s)", "host_cpus": os.cpu_count()}


def run_mine(args):
    import torch
    from mla_latent_kv_45_b200 import _lib as L
    from mla_latent_kv_45_b200 import build, synth
    from mla_latent_kv_45_b200.layer import DecodeLayer

    rank, world, local = setup_dist(args)
    torch.cuda.set_device(local)
    build.build()
    wl = workload(args.workload, rank)
    assert wl.new_tokens == 1, "the bench runs whole decode steps"
    W = synth.make_weights(wl)
    prior = synth.make_prior_lengths(wl)
    pc = synth.make_paged_cache(wl, prior)
    h = synth.make_hidden(wl)
    lens = prior + 1
    dims = L.Dims(wl.n_heads, wl.d_c, wl.d_rope, wl.d_nope, wl.d_v, wl.page_size, L.MLA_BF16,
                  wl.rope_layout, wl.rope_base, wl.rms_eps)
    dev = torch.device("cuda", local)
    Wd = {k: (None if v is None else torch.from_numpy(v).to(dev).to(torch.bfloat16))
          for k, v in W.items()}
    pool = torch.from_numpy(pc.pool.view(np.int16)).to(dev).view(torch.bfloat16)
    cache = L.PagedCache(pool, torch.from_numpy(pc.block_table).to(dev),
                         torch.from_numpy(lens.astype(np.int32)).to(dev))
    hd = torch.from_numpy(h).to(dev).to(torch.bfloat16)
    pos = torch.from_numpy(prior.astype(np.int32)).to(dev)
    layer = DecodeLayer(dims, Wd, wl.batch, args.num_splits, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        layer.step(cache, hd, pos)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = layer.device_error()
    if st != 0:
        raise RuntimeError(f"device error {L.STATUS.get(st)} during warm-up")

    # per-call events inside the timed region: the append on the layer's side
    # stream, the other calls on the main stream (see DecodeLayer.step)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]

    def timed_step(e):
        layer.step(cache, hd, pos, stream, e)

    gpu_id = torch.cuda.get_device_properties(dev).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else gpu_id
    clocks = ClockSampler(gpu_id) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.5)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        timed_step(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    elapsed = start.elapsed_time(end)  # ms
    per_call = np.array([[e[0].elapsed_time(e[1]), e[2].elapsed_time(e[3]),
                          e[4].elapsed_time(e[5]), e[5].elapsed_time(e[6])] for e in ev])
    st = layer.device_error()
    if st != 0:
        raise RuntimeError(f"device error {L.STATUS.get(st)} in the timed region")
    if clocks:
        clocks.stop()

    # end-to-end through the public API with host buffers: pinned h2d of the
    # step's inputs and d2h of its output inside the timed region
    h_host = hd.cpu().pin_memory()
    pos_host = pos.cpu().pin_memory()
    lens_host = cache.seq_lens.cpu().pin_memory()
    out_host = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    for _ in range(max(3, args.warmup // 4)):
        hd.copy_(h_host, non_blocking=True)
        step()
        out_host.copy_(layer.out, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(args.steps):
        hd.copy_(h_host, non_blocking=True)
        pos.copy_(pos_host, non_blocking=True)
        cache.seq_lens.copy_(lens_host, non_blocking=True)
        step()
        out_host.copy_(layer.out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    elapsed, e2e_ms, attn_ms_total = max_over_ranks([elapsed, e2e_ms, per_call[:, 2].sum()],
                                                    world, dev)

    alg = algorithmic(wl, lens)
    hbm, tf, tf_sus, src = peaks()
    ms_step = elapsed / args.steps
    value = alg["rows"] * wl.n_heads * world / (ms_step / 1e3)
    attn_ms = attn_ms_total / args.steps
    t_bytes = alg["attn_bytes"] / (hbm * 1e9)
    t_flops = alg["attn_flops"] / (tf * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    if bound == "hbm":
        achieved, peak, unit = alg["attn_bytes"] / (attn_ms / 1e3) / 1e9, hbm, "GB/s"
    else:
        achieved, peak, unit = alg["attn_flops"] / (attn_ms / 1e3) / 1e12, tf, "TFLOP/s"
    traffic = stored_traffic(wl.name.split("+")[0])
    step_t = max(alg["step_bytes"] / (hbm * 1e9), alg["step_flops"] / (tf * 1e12))
    h2d = (hd.numel() * hd.element_size() + pos.numel() * 4 + cache.seq_lens.numel() * 4)
    d2h = layer.out.numel() * layer.out.element_size()
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(wl, lens), "batch_per_gpu": wl.batch,
                   "global_batch": wl.batch * world, "cached_rows_per_step": alg["rows"],
                   "parallelism": f"dp{world} (sequences sharded, no collective)",
                   "l2": "no flush: per-step inputs (cache %.0f MB + weights %.0f MB) exceed the "
                         "126 MB L2" % (alg["rows"] * ROW_BYTES / 1e6, 2 * alg["params"] / 1e6),
                   "num_splits": args.num_splits},
        "roofline": {"kernel": "mla_decode_attn (plan + attention + split merge)",
                     "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic, "peak_source": src,
                     "algorithmic_bytes": alg["attn_bytes"], "algorithmic_flops": alg["attn_flops"],
                     "ms_per_launch": attn_ms},
        "step_roofline": {"bytes": alg["step_bytes"], "flops": alg["step_flops"],
                          "roofline_ms": step_t * 1e3, "frac": step_t * 1e3 / ms_step},
        "breakdown_ms": dict(zip(["cache_append", "absorb_q", "decode_attn", "unabsorb_out"],
                                 [float(x) for x in per_call.mean(0)])),
        "e2e": {"value": alg["rows"] * wl.n_heads * world / (e2e_ms / args.steps / 1e3),
                "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    if rank == 0:
        res["clocks"] = clocks.summary(t_wall0, t_wall1) if clocks else None
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_sample(wl, W, pc, h, lens)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# Launches of this library per decode step (checked against the ncu launch list):
# append 2 (W_DKV+W_KR projection, RMSNorm/RoPE/page write), absorb_q 5 (W_DQ,
# its split-K reduce, W_UQ+W_QR, W_UK, RoPE), decode_attn 3 (plan, attention,
# merge), unabsorb_out 3 (W_UV, W_O, its split-K reduce).
LAUNCHES_PER_STEP = 13


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
    import oracle
    from mla_latent_kv_45_b200 import synth
    wl = workload(args.workload, 0)
    W = synth.make_weights(wl)
    prior = synth.make_prior_lengths(wl)
    pc = synth.make_paged_cache(wl, prior)
    h = synth.make_hidden(wl)
    od = oracle.Dims(n_heads=wl.n_heads, d_c=wl.d_c, d_rope=wl.d_rope, d_nope=wl.d_nope,
                     d_v=wl.d_v, rope_base=wl.rope_base, rms_eps=wl.rms_eps,
                     rope_layout=wl.rope_layout)
    # size each step's sample so the whole run stays within ~2 minutes
    t = time.perf_counter()
    oracle.decode_step(h[:1], [pc.rows_f32(0, 63)], W, od)
    per_row = (time.perf_counter() - t) / 64
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(prior[0] + 1, max(16, budget / max(per_row, 1e-9))))
    rows = [pc.rows_f32(b % wl.batch, n - 1) for b in range(wl.batch)]

    def one(k):
        b = k % wl.batch
        oracle.decode_step(h[b:b + 1], [rows[b]], W, od)

    for k in range(args.warmup):
        one(k)
    t0 = time.perf_counter()
    for k in range(args.steps):
        one(k)
    dt = time.perf_counter() - t0
    value = n * wl.n_heads * args.steps / dt
    try:
        import threadpoolctl
        threads = max((p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        threads = 1
    sample = (f"each step: one sequence of {wl.name} (cycling over its {wl.batch}), first {n} "
              f"cached rows incl. the new token, all {wl.n_heads} heads, whole un-absorbed fp64 "
              f"decode step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": describe(wl, prior + 1)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(threads), "kind": "oracle",
                         "sample": sample, "host_cpus": os.cpu_count()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", default="v2_batch64")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mine(args)


if __name__ == "__main__":
    main()
