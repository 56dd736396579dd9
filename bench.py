"""Benchmark of the deferred-RoPE paged attention hot path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload decode_8b] [--no-prefill] [--no-compare] [--no-e2e] [--no-cpu]
                [--extended] [--cache-sim] [--profile-case NAME]

One step (ours) = one pass of the hot path over one batch of the decode
workload with Llama-3.1-8B attention shapes (64 requests, 32/8 heads, d 128,
8 Zipf(1.0) documents of 512 tokens from a 1000-document pool plus a 64-token
question; one decode token each): lazy_kv_write of the 64 new tokens, then
lazy_decode_attn (split-K attention + combine).  The pool of cached documents
is resident in HBM before timing starts, as in serving.  `value` is logical
decode K/V bytes per second over all ranks (every visible key and value of
every request, once).  L2 (126 MB) is flushed between timed steps by writing
a 512 MiB buffer outside the timed intervals.

Also measured in the same run and reported in sub-objects:
  prefill     the causal prefill workload with 8B shapes (16 requests x 256
              query tokens over 10 documents), TFLOP/s over visible pairs;
  comparison  the position-aware alternative on the same inputs: materialise
              re-rotated keys, then plain paged attention; also the rotation-off
              kernel, and the same attention with ALiBi in place of RoPE (timing
              only);
  e2e         the decode metric through the same C-ABI calls with the step's
              inputs copied from pinned host memory and the output copied back
              inside the timed region;
  cpu_baseline  the fp64 oracle on a bounded sample of requests, host cores.

--impl reference times the fp64 CPU oracle itself (the only reference
implementation this project has) on a bounded sample of the same workload.
Multi-GPU: one independent replica per rank (the path needs no exchange step);
the time is the maximum over ranks and the work the sum over ranks.

--extended adds decode at 70B shapes (Zipf 1.2 and uniform popularity) and the
mixed 8B serving step (GQA and MQA), with the whole step timed as two calls
and as one lazy_mixed_attn call.  --cache-sim runs the host-side cache-hit
simulation of position-agnostic, position-aware and prefix caching (no GPU).
--profile-case launches only the attention kernel of a small case (or of
the mixed 8B MQA step's decode batch), for profiler captures.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode KV GB/s & prefill TFLOP/s on 1 B200, % of roofline; oracle ×"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernels from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the SHA-256 of the
# kernel source it was taken on; reported as null when the source changed.
# Each figure holds for the kernel source whose hash it carries; a source edit voids it, except an
# edit of comments alone (same lines), after which the hash is re-pinned.
TRAFFIC = {
    # ncu --clock-control none --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
    #     -k regex:decode_split -s 3 -c 1
    #     python bench.py --steps 2 --warmup 3 --no-cpu --no-compare --no-e2e --no-distinct
    "decode_8b": {"sha": "b4ca7d6410749acd", "bytes": 786105600 + 7165184},
    # the same command with --no-prefill --workload decode_8b_distinct
    "decode_8b_distinct": {"sha": "b4ca7d6410749acd", "bytes": 1095527424 + 6870272},
    # the first command with -k regex:prefill_tc
    "prefill_8b": {"sha": "048840e346fb33b7", "bytes": 302145280 + 26523392},
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha(name: str) -> str:
    path = os.path.join(ROOT, "position_agnostic_paged_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(key: str, src: str, scale: float = 1.0):
    t = TRAFFIC.get(key)
    if not t or t["sha"] != kernel_sha(src):
        return None
    return t["bytes"] * scale


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus: int):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _all_reduce(world, x: float, op_name: str) -> float:
    """x reduced over the ranks (timings and counts only; the path itself exchanges nothing).
    The tensor lives where the process group's backend wants it: the GPU for NCCL, the host for
    gloo (the multi-rank logic is tested on CPU with gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(world, x: float) -> float:
    return _all_reduce(world, x, "MAX")


def sum_over_ranks(world, x: float) -> float:
    return _all_reduce(world, x, "SUM")


def whole_job(world, local_units: float, local_ms: float):
    """Whole-job throughput of independent replicas: the units all ranks processed divided by the
    slowest rank's time.  Returns (units per second, that time in ms)."""
    ms = max_over_ranks(world, local_ms)
    units = sum_over_ranks(world, float(local_units))
    return units / (ms * 1e-3), ms


# ----------------------------------------------------------------------------- timing helpers
class L2Flush:
    def __init__(self):
        import torch

        self.buf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def timed_steps(run_step, steps: int, warmup: int, flush, world, inner=None):
    """Runs warmup + steps; returns (total device ms over the timed steps, per-launch ms of `inner`).

    Each timed step is bracketed by CUDA events on the current stream; the L2
    flush runs between steps outside the events.  `inner` (optional) is a
    pair of event lists filled by run_step around the dominant launch.
    """
    import torch

    for _ in range(warmup):
        flush()
        run_step(None)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    inner_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        starts[i].record()
        run_step(inner_ev[i])
        ends[i].record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    total = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    inner_ms = [a.elapsed_time(b) for a, b in inner_ev] if inner else None
    return total, inner_ms


# ----------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch

    from position_agnostic_paged_b200 import accounting
    from position_agnostic_paged_b200 import lazy_attn as la
    from position_agnostic_paged_b200 import workloads as W
    from position_agnostic_paged_b200.runner import DevicePool, DeviceStep

    world, rank, local = dist_setup(args.gpus)
    peaks, peak_src = load_peaks()
    flush = L2Flush()

    # ---------------------------------------------------------------- decode (headline)
    t0 = time.time()
    wl = W.make(args.workload)
    step = [s for s in wl.steps if s.kind == "decode"][0]
    pool = DevicePool(wl).setup()
    ds = DeviceStep(pool, step, with_plain=not args.no_compare)
    torch.cuda.synchronize()
    log(f"[rank {rank}] decode workload ready in {time.time() - t0:.1f}s: {step.num_req} requests, "
        f"{int(step.kv_len.sum())} keys, pool {wl.num_blocks} blocks")
    dec_bytes = accounting.decode_kv_bytes(step.kv_len, wl.hkv, wl.d)

    def decode_step(ev):
        ds.write_new_tokens_dev()
        if ev is not None:
            ev[0].record()
        ds.attend()
        if ev is not None:
            ev[1].record()

    # the new tokens' K/V are uploaded once; each step rewrites the same slots
    _prepare_step_writes(ds)
    clocks = ClockSampler(local)
    clocks.start()
    total_ms, attn_ms = timed_steps(decode_step, args.steps, args.warmup, flush, world, inner=True)
    clk = clocks.stop()
    rate, ms_step = whole_job(world, dec_bytes, total_ms / args.steps)
    attn_avg = max_over_ranks(world, float(np.mean(attn_ms)))
    value = rate / 1e9
    achieved = dec_bytes / (attn_avg * 1e-3) / 1e9
    if pool.status() != 0:
        raise SystemExit(f"device status {pool.status()} after decode steps")

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: Llama-3.1-8B attention shapes (Hq 32, Hkv 8, d 128), "
                               f"{step.num_req} requests x {int(step.kv_len[0])} keys (8 Zipf(1.0) docs x 512 "
                               "+ 64-token question + 1 decode token), 1000-doc pool",
                   "global_batch": step.num_req * world, "seq_len": int(step.kv_len.max()),
                   "parallelism": f"replicas x{world}", "l2": "flushed between timed steps (512 MiB write)",
                   "step": "lazy_kv_write(new tokens) + lazy_decode_attn"},
        "roofline": {"bound": "hbm", "kernel": "lazy_decode_attn (split-K attention + combine)",
                     "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": peak_src,
                     "traffic": traffic_for("decode_8b", "decode.cu"),
                     "algorithmic_bytes_per_launch": dec_bytes},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }

    # ---------------------------------------------------------------- comparison paths on the same inputs
    if not args.no_compare:
        def plain_step(ev):
            if ev is not None:
                ev[0].record()
            ds.attend_plain()
            if ev is not None:
                ev[1].record()

        def mat_step(ev):
            ds.materialize()
            ds.attend_plain()

        ds.materialize()
        plain_total, _ = timed_steps(plain_step, args.steps, args.warmup, flush, world)
        mat_total, _ = timed_steps(mat_step, args.steps, args.warmup, flush, world)
        torch.cuda.synchronize()
        lazy_vs_plain = float((ds.out.float() - ds.out_plain.float()).abs().max().item())
        alibi_total = _time_alibi(ds, args, flush, world)
        result["comparison"] = {
            "lazy_decode_attn_ms": round(attn_avg, 5),
            "plain_decode_attn_ms": round(max_over_ranks(world, plain_total / args.steps), 5),
            "materialize_then_attend_ms": round(max_over_ranks(world, mat_total / args.steps), 5),
            "materialized_k_bytes": int(ds.k_mat.numel() * 2),
            "max_abs_lazy_minus_plain": lazy_vs_plain,
            "alibi_decode_attn_ms": round(max_over_ranks(world, alibi_total / args.steps), 5),
        }
        result["gpu_launches"] += 2 * args.steps + 3 * args.steps + 2 * args.steps

    # ---------------------------------------------------------------- e2e through the public API
    if not args.no_e2e:
        result["e2e"] = run_e2e(ds, pool, step, dec_bytes, args, world)
        result["gpu_launches"] += 3 * args.steps

    del ds, pool
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- decode with no shared documents
    if not args.no_distinct:
        result["decode_distinct"] = run_decode_distinct(args, world, peaks, peak_src, flush)
        result["gpu_launches"] += 3 * args.steps

    # ---------------------------------------------------------------- prefill leg
    if not args.no_prefill:
        result["prefill"] = run_prefill(args, world, peaks, peak_src, flush)
        result["gpu_launches"] += result["prefill"].pop("_launches")

    # ---------------------------------------------------------------- other workloads (optional)
    if args.extended:
        result["extended"] = run_extended(args, world, peaks, peak_src, flush)

    # ---------------------------------------------------------------- CPU baseline (oracle), rank 0, N = 1
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(wl, step, args.cpu_requests)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def _prepare_step_writes(ds):
    """Uploads the step's new-token K/V once, so that timed steps rewrite the
    same slots from device memory (the pool write is part of the step)."""
    import torch

    from position_agnostic_paged_b200 import lazy_attn as la

    wl, rows, dev = ds.pool.wl, ds.write_rows, ds.pool.device
    ds.wk = torch.from_numpy(np.ascontiguousarray(wl.k_store[rows]).view(np.int16)).to(dev).view(torch.bfloat16)
    ds.wv = torch.from_numpy(np.ascontiguousarray(wl.v_store[rows]).view(np.int16)).to(dev).view(torch.bfloat16)
    ds.wslot = torch.from_numpy(wl.store_slot[rows].astype(np.int32)).to(dev)
    ds.wj = torch.from_numpy(wl.store_j[rows].astype(np.int32)).to(dev)

    def write_dev(stream=None):
        p = ds.pool
        la.kv_write(ds.cfg, ds.wk, ds.wv, ds.wslot, ds.wj, p.k_pool, p.v_pool, p.blk_meta, p.d_status, stream)

    ds.write_new_tokens_dev = write_dev


def run_e2e(ds, pool, step, dec_bytes, args, world):
    """Decode metric with the step's inputs in pinned host memory: H2D copies,
    lazy_kv_write, lazy_decode_attn and the D2H copy of the output, all timed."""
    import torch

    from position_agnostic_paged_b200 import lazy_attn as la

    wl = pool.wl
    rows = ds.write_rows

    def pinned(a: np.ndarray, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).view(dt).pin_memory()

    h = {
        "q": pinned(step.q_raw.view(np.int16), torch.int16),
        "qpos": pinned(step.q_pos.astype(np.int32), torch.int32),
        "table": pinned(ds.words_np.view(np.int32), torch.int32),
        "indptr": pinned(step.table_indptr.astype(np.int32), torch.int32),
        "k": pinned(wl.k_store[rows].view(np.int16), torch.int16),
        "v": pinned(wl.v_store[rows].view(np.int16), torch.int16),
        "slot": pinned(wl.store_slot[rows].astype(np.int32), torch.int32),
        "j": pinned(wl.store_j[rows].astype(np.int32), torch.int32),
    }
    d = {k: torch.empty_like(v, device="cuda") for k, v in h.items()}
    out_h = torch.empty(ds.out.shape, dtype=torch.int16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = out_h.numel() * 2
    flush = L2Flush()

    def e2e_step(ev):
        for k in h:
            d[k].copy_(h[k], non_blocking=True)
        la.kv_write(ds.cfg, d["k"].view(torch.bfloat16), d["v"].view(torch.bfloat16), d["slot"], d["j"],
                    pool.k_pool, pool.v_pool, pool.blk_meta, pool.d_status)
        la.decode_attn(ds.cfg, d["q"].view(torch.bfloat16), d["qpos"], d["table"], d["indptr"], ds.max_words,
                       pool.blk_meta, pool.k_pool, pool.v_pool, ds.out, ds.workspace, pool.d_status)
        out_h.copy_(ds.out.view(torch.int16), non_blocking=True)

    total, _ = timed_steps(e2e_step, args.steps, args.warmup, flush, world)
    rate, ms = whole_job(world, dec_bytes, total / args.steps)
    return {"value": round(rate / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


def run_decode_distinct(args, world, peaks, peak_src, flush):
    """The decode 8B step with no document shared across requests (512 distinct documents, 8 per
    request): every logical K/V byte is a distinct byte in HBM, so L2 cannot serve repeats and the
    logical-byte fraction of the HBM peak is the kernel's real HBM efficiency."""
    from position_agnostic_paged_b200 import accounting
    from position_agnostic_paged_b200 import workloads as W
    from position_agnostic_paged_b200.runner import DevicePool, DeviceStep

    wl = W.make("decode_8b_distinct")
    step = wl.steps[0]
    pool = DevicePool(wl).setup()
    ds = DeviceStep(pool, step)
    _prepare_step_writes(ds)
    b = accounting.decode_kv_bytes(step.kv_len, wl.hkv, wl.d)

    def st(ev):
        ds.write_new_tokens_dev()
        if ev is not None:
            ev[0].record()
        ds.attend()
        if ev is not None:
            ev[1].record()

    total, inner = timed_steps(st, args.steps, args.warmup, flush, world, inner=True)
    attn = max_over_ranks(world, float(np.mean(inner)))
    if pool.status() != 0:
        raise SystemExit(f"device status {pool.status()} after distinct-document decode steps")
    gbs = b / (attn * 1e-3) / 1e9
    return {"workload": "decode_8b_distinct: decode 8B shapes, 64 requests x 4161 keys, 8 documents per request "
                        "drawn without replacement across the batch (no document shared)",
            "kv_bytes": b, "attn_ms": round(attn, 5), "GB/s": round(gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peak_src,
                         "traffic": traffic_for("decode_8b_distinct", "decode.cu")}}


def _time_alibi(ds, args, flush, world) -> float:
    """The step's attention with ALiBi (the model's slopes for its query heads) in place of RoPE,
    on the same pool and inputs: the cost of the other relative encoding.  Timing only (the pool
    holds RoPE keys, so the values are not compared here; the parity tests check ALiBi)."""
    import dataclasses

    from position_agnostic_paged_b200.rope import alibi_slopes
    rope_cfg = ds.cfg
    ds.cfg = dataclasses.replace(rope_cfg, alibi_slopes=alibi_slopes(rope_cfg.num_q_heads))
    try:
        total, _ = timed_steps(lambda ev: ds.attend(out=ds.out_plain), args.steps, args.warmup, flush, world)
    finally:
        ds.cfg = rope_cfg
    return total


def run_prefill(args, world, peaks, peak_src, flush):
    import torch

    from position_agnostic_paged_b200 import accounting
    from position_agnostic_paged_b200 import lazy_attn as la
    from position_agnostic_paged_b200 import workloads as W
    from position_agnostic_paged_b200.runner import DevicePool, DeviceStep

    wl = W.make("prefill_8b")
    step = wl.steps[0]
    pool = DevicePool(wl).setup()
    ds = DeviceStep(pool, step, with_plain=not args.no_compare)
    _prepare_step_writes(ds)
    flops = accounting.prefill_flops(step.visible_pairs, wl.hq, wl.d)

    def pf_step(ev):
        ds.write_new_tokens_dev()
        if ev is not None:
            ev[0].record()
        ds.attend()
        if ev is not None:
            ev[1].record()

    total, attn = timed_steps(pf_step, args.steps, args.warmup, flush, world, inner=True)
    rate, ms = whole_job(world, flops, total / args.steps)
    attn_avg = max_over_ranks(world, float(np.mean(attn)))
    if pool.status() != 0:
        raise SystemExit(f"device status {pool.status()} after prefill steps")
    achieved = flops / (attn_avg * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    comparison = None
    if not args.no_compare:
        # the same chunk through the comparison paths: rotation off (keys materialised once,
        # outside the timing), and materialise-then-attend (the materialisation timed too)
        def plain_step(ev):
            ds.attend_plain()

        def mat_step(ev):
            ds.materialize()
            ds.attend_plain()

        ds.materialize()
        plain_total, _ = timed_steps(plain_step, args.steps, args.warmup, flush, world)
        mat_total, _ = timed_steps(mat_step, args.steps, args.warmup, flush, world)
        torch.cuda.synchronize()
        comparison = {
            "lazy_prefill_attn_ms": round(attn_avg, 5),
            "plain_prefill_attn_ms": round(max_over_ranks(world, plain_total / args.steps), 5),
            "materialize_then_attend_ms": round(max_over_ranks(world, mat_total / args.steps), 5),
            "materialized_k_bytes": int(ds.k_mat.numel() * 2),
            "max_abs_lazy_minus_plain": float((ds.out.float() - ds.out_plain.float()).abs().max().item()),
        }
        alibi_total = _time_alibi(ds, args, flush, world)
        comparison["alibi_prefill_attn_ms"] = round(max_over_ranks(world, alibi_total / args.steps), 5)
    # attention launches per call: the prefill kernel, plus the combine kernel when the workspace
    # lets the last wave's units run split
    per_call = 2 if ds.workspace.numel() >= 16 and la.prefill_workspace_bytes(
        ds.cfg, step.num_req, step.total_q, ds.max_q, ds.max_words) > 0 else 1
    launches = (1 + per_call) * args.steps + ((per_call + 1 + per_call + per_call) * args.steps if comparison else 0)
    return {
        "_launches": launches,
        "workload": "prefill_8b: Llama-3.1-8B shapes, 16 requests x 256 causal query tokens over 10 Zipf(1.0) "
                    "docs x 512 (5376 keys), 1000-doc pool",
        "value": round(rate / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
        "step": "lazy_kv_write(256-token chunks) + lazy_prefill_attn",
        "algorithmic_flops_per_launch": flops,
        "roofline": {"bound": "tensor", "kernel": "lazy_prefill_attn", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "traffic": traffic_for("prefill_8b", "prefill_tc.cu")},
        **({"comparison": comparison} if comparison else {}),
    }


def _pf_calls(ds) -> int:
    """Launches of one prefill attention call: the kernel, and the combine kernel when the
    workspace lets the last wave's units run split."""
    from position_agnostic_paged_b200 import lazy_attn as la
    st = ds.step
    return 2 if ds.workspace.numel() >= 16 and la.prefill_workspace_bytes(
        ds.cfg, st.num_req, st.total_q, ds.max_q, ds.max_words) > 0 else 1


def run_extended(args, world, peaks, peak_src, flush):
    """Decode 70B shapes (Zipf 1.2 and uniform popularity) and the mixed 8B serving
    step (32 prefill chunks + 192 decodes, 1 GiB pool; GQA and MQA): per step
    kind, the attention time and its throughput against the roofline."""
    import torch

    from position_agnostic_paged_b200 import accounting
    from position_agnostic_paged_b200 import workloads as W
    from position_agnostic_paged_b200.runner import DevicePool, DeviceStep, mixed_attend

    out = {}
    for name in ("decode_70b", "decode_70b_uniform", "mixed_8b", "mixed_8b_mqa"):
        t0 = time.time()
        wl = W.make(name)
        pool = DevicePool(wl).setup()
        entry = {"unique_docs": wl.info["unique_docs_used"], "pool_blocks": wl.num_blocks}
        kept = {}
        for step in wl.steps:
            ds = DeviceStep(pool, step)
            _prepare_step_writes(ds)

            def st(ev):
                ds.write_new_tokens_dev()
                if ev is not None:
                    ev[0].record()
                ds.attend()
                if ev is not None:
                    ev[1].record()

            total, inner = timed_steps(st, args.steps, args.warmup, flush, world, inner=True)
            attn = max_over_ranks(world, float(np.mean(inner)))
            if step.kind == "decode":
                b = accounting.decode_kv_bytes(step.kv_len, wl.hkv, wl.d)
                entry["decode"] = {"requests": step.num_req, "kv_bytes": b, "attn_ms": round(attn, 5),
                                   "GB/s": round(b / (attn * 1e-3) / 1e9, 1),
                                   "frac_of_hbm_peak": round(b / (attn * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
            else:
                f = accounting.prefill_flops(step.visible_pairs, wl.hq, wl.d)
                tf = f / (attn * 1e-3) / 1e12
                entry["prefill"] = {"requests": step.num_req, "flops": f, "attn_ms": round(attn, 5),
                                    "TFLOP/s": round(tf, 1),
                                    "frac_of_bf16_peak": round(tf / peaks.get("bf16_tflops", 1590.0), 4)}
            kept[step.kind] = ds
        if "prefill" in kept and "decode" in kept:
            # the whole serving step: the two attention calls back to back on one stream, and the
            # same two batches in one lazy_mixed_attn call
            pf, dc = kept["prefill"], kept["decode"]

            def seq(ev):
                pf.attend()
                dc.attend()

            def mixed(ev):
                mixed_attend(pf, dc)

            seq_total, _ = timed_steps(seq, args.steps, args.warmup, flush, world)
            mix_total, _ = timed_steps(mixed, args.steps, args.warmup, flush, world)
            entry["step"] = {"sequential_ms": round(max_over_ranks(world, seq_total / args.steps), 5),
                             "lazy_mixed_attn_ms": round(max_over_ranks(world, mix_total / args.steps), 5)}
            launches_extra = (_pf_calls(pf) + 2) * 2 * args.steps
            entry["step"]["gpu_launches"] = launches_extra
        del kept, ds
        if pool.status() != 0:
            raise SystemExit(f"device status {pool.status()} in {name}")
        del pool
        torch.cuda.empty_cache()
        log(f"[extended] {name} done in {time.time() - t0:.1f}s")
        out[name] = entry
    return out


def cpu_baseline(wl, step, n_req: int):
    import oracle
    from position_agnostic_paged_b200 import accounting

    n_req = min(n_req, step.num_req)
    sel_q = np.repeat(np.arange(n_req, dtype=np.int32), wl.hq)
    sel_h = np.tile(np.arange(wl.hq, dtype=np.int32), n_req)
    t0 = time.perf_counter()
    oracle.attend(num_q_heads=wl.hq, num_kv_heads=wl.hkv, rope_base=wl.rope_base, q_raw=step.q_raw,
                  cu_q=step.cu_q, q_pos=step.q_pos, seg_indptr=step.seg_indptr, seg_src=step.seg_src,
                  seg_off=step.seg_off, seg_len=step.seg_len, k_tok=wl.k_store, v_tok=wl.v_store,
                  sel_q=sel_q, sel_h=sel_h)
    dt = time.perf_counter() - t0
    b = accounting.decode_kv_bytes(step.kv_len[:n_req], wl.hkv, wl.d)
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_req} of {step.num_req} decode requests, all {wl.hq} heads ({dt:.1f} s)"}


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from position_agnostic_paged_b200 import accounting
    from position_agnostic_paged_b200 import workloads as W

    wl = W.make(args.workload)
    step = [s for s in wl.steps if s.kind == "decode"][0]
    n_req = max(1, args.ref_requests)

    def one(i):
        r = np.arange(i * n_req, (i + 1) * n_req) % step.num_req
        sel_q = np.repeat(r.astype(np.int32), wl.hq)
        sel_h = np.tile(np.arange(wl.hq, dtype=np.int32), r.size)
        oracle.attend(num_q_heads=wl.hq, num_kv_heads=wl.hkv, rope_base=wl.rope_base, q_raw=step.q_raw,
                      cu_q=step.cu_q, q_pos=step.q_pos, seg_indptr=step.seg_indptr, seg_src=step.seg_src,
                      seg_off=step.seg_off, seg_len=step.seg_len, k_tok=wl.k_store, v_tok=wl.v_store,
                      sel_q=sel_q, sel_h=sel_h)
        return accounting.decode_kv_bytes(step.kv_len[r], wl.hkv, wl.d)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    total_bytes = 0
    for i in range(args.steps):
        total_bytes += one(args.warmup + i)
    dt = time.perf_counter() - t0
    value = total_bytes / dt / 1e9
    sample = f"{n_req} of {step.num_req} decode requests per step, all {wl.hq} heads"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload} (bounded sample: {sample})", "global_batch": n_req,
                   "seq_len": int(step.kv_len.max()), "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """A case for profiler captures: 2 prefill requests (64 CTAs) or 8 decode requests of the 8B
    shapes over a 100-document pool, or 32 decode requests of the MQA shapes (Hq 32, Hkv 1) over a
    400-document pool; or the whole decode batch of the mixed 8B MQA step (192 requests, 1 GiB
    pool), for one-pass counters only; the attention kernel launched --steps times."""
    import torch
    from position_agnostic_paged_b200 import workloads as W
    from position_agnostic_paged_b200.runner import DevicePool, DeviceStep
    if args.profile_case == "prefill_small":
        wl = W.make("prefill_8b", n_docs=100, n_prefill=2)
    elif args.profile_case == "decode_small":
        wl = W.make("decode_8b", n_docs=100, n_decode=8)
    elif args.profile_case == "decode_mqa_small":
        wl = W.make("mixed_8b_mqa", n_docs=400, n_prefill=0, n_decode=32)
    else:
        wl = W.make("mixed_8b_mqa")   # its decode step only
    pool = DevicePool(wl).setup()
    ds = DeviceStep(pool, [st for st in wl.steps if st.kind == ("prefill" if "prefill" in args.profile_case
                                                                    else "decode")][0])
    ds.write_new_tokens()
    for _ in range(args.steps):
        ds.attend()
    torch.cuda.synchronize()
    log(f"[profile-case] {args.profile_case}: {args.steps} launches, status {pool.status()}")


def run_cache_sim(args):
    """Cache-hit ratios of position-agnostic caching against position-aware (re-encoding and
    exact-offset) and prefix caching, at a 1 GB KV budget of Llama-3.1-8B geometry, for three Zipf
    exponents of document popularity (documents in random order, then ordered by popularity rank),
    then across budgets from 128 MB to 8 GB at Zipf 1.0; host only, one JSON line per exponent or
    budget."""
    from position_agnostic_paged_b200 import cache_sim
    t0 = time.perf_counter()
    n_sweep = max(1, args.cache_requests * 3 // 10)
    for row in cache_sim.compare(n_requests=args.cache_requests):
        print(json.dumps({"metric": "cache_hit_ratio", "unit": "fraction of document blocks",
                          "data": "synthetic", "requests": args.cache_requests, **row}), flush=True)
    for row in cache_sim.compare(n_requests=n_sweep, order="rank"):
        print(json.dumps({"metric": "cache_hit_ratio", "unit": "fraction of document blocks",
                          "data": "synthetic", "requests": n_sweep, **row}), flush=True)
    for row in cache_sim.budget_sweep(n_requests=n_sweep):
        print(json.dumps({"metric": "cache_hit_ratio", "unit": "fraction of document blocks",
                          "data": "synthetic", "requests": n_sweep, "sweep": "budget", **row}), flush=True)
    log(f"[cache-sim] {time.perf_counter() - t0:.1f} s")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_8b")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-compare", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-distinct", action="store_true",
                    help="skip the decode step over documents shared by no two requests")
    ap.add_argument("--extended", action="store_true",
                    help="also time decode 70B (Zipf 1.2 and uniform) and the mixed 8B step (GQA, MQA)")
    ap.add_argument("--profile-case", choices=["prefill_small", "decode_small", "decode_mqa_small", "decode_mqa_full"],
                    help="launch only the attention kernel of a small case --steps times (for ncu captures; "
                         "prints no result line)")
    ap.add_argument("--cache-sim", action="store_true",
                    help="host-side cache-hit simulation of the caching policies (no GPU; prints one line "
                         "per Zipf exponent)")
    ap.add_argument("--cache-requests", type=int, default=20000)
    ap.add_argument("--cpu-requests", type=int, default=64)
    ap.add_argument("--ref-requests", type=int, default=2)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.cache_sim:
        run_cache_sim(args)
    elif args.profile_case:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
