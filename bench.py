#!/usr/bin/env python3
"""Benchmark of the chunk-causal attention layer on B200.

One step = one pass of the whole layer over one chunk: ``unstep_rope_kv_append`` (3D RoPE +
ring-buffer KV append) followed by ``unstep_window_attn`` (attention over the window).  The
default workload is the Wan-1.3B-shaped layer with a full causal cache: 12 heads x 128,
30x52 = 1560 tokens per latent frame, a chunk of 3 frames (4680 queries) attending all 21 frames
of a 5-s clip (32760 keys); the cache is filled by streaming chunks 0..6 first, and each timed
step is a re-forward of the last chunk (the next denoising step).

Output: one JSON line.  ``value`` = attention FLOPs (4*B*H*L*Lk*D, true keys) of all ranks per
second of step time (device-timed with CUDA events, max over ranks, L2 flushed between steps);
``e2e`` = the same metric through the public API from pinned host buffers (host->device copy of
q/k/v and device->host copy of the output inside the timed region).

``--impl reference`` times the fp64 CPU oracle (rank 0 only) on a bounded sample of the same
workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "windowed-attn TFLOP/s & chunk-steps/s at Wan-1.3B shape; % bf16/HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------------------------
# helpers shared with the tests (no GPU needed)
# ----------------------------------------------------------------------------------------------

def dist_env():
    """(rank, local_rank, world) from torchrun's environment; (0, 0, 1) when run directly."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rank_seed(base: int, rank: int) -> int:
    """Each rank streams its own independent video stream (weak scaling, no exchange)."""
    return base + 7919 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a per-rank time (the job takes as long as its slowest rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:  # noqa: BLE001
        return dict(FALLBACK_PEAKS), "fallback"


ATTN_SOURCES = ("window_attn.cu", "sm100.cuh", "internal.h", "limits.h")
ROPE_SOURCES = ("rope_append.cu", "internal.h", "limits.h")
GEMM_SOURCES = ("gemm2sm.cu", "sm100.cuh", "gemm.h", "limits.h")
CONV_SOURCES = ("conv3d.cu", "sm100.cuh", "conv3d.h", "limits.h")


def source_digest(names=ATTN_SOURCES) -> str:
    """Digest of a kernel's source files, as the ncu summaries in profiles/ record it."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "causal_video_diffusion_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_source_digest() -> str:
    return source_digest(ATTN_SOURCES)


def profile_traffic(profile: str, names):
    """DRAM bytes per launch recorded in profiles/<profile>, if it was taken on the current
    source of the kernel (else None)."""
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)\s+source:\s*([0-9a-f]+)", text)
    if not m or m.group(2) != source_digest(names):
        return None
    return float(m.group(1))


def profiled_traffic(workload: str, rope_q: bool = False):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current kernel source (else None); ``rope_q``: the instantiation with the query prologue."""
    name = f"window_attn_qrope_{workload}.txt" if rope_q else f"window_attn_{workload}.txt"
    return profile_traffic(name, ATTN_SOURCES)


CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
CLOCK_INTERVAL_MS = 50
CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def summarize_clocks(lines, t0, t1):
    """Median SM clock, maximum clock and active throttle reasons of the nvidia-smi samples taken
    between wall times t0 and t1 (seconds; the timed region), widened by one sampling interval.
    A region shorter than the interval may hold no sample: then the sample nearest to its middle
    stands for it, and ``window`` says so."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            rows.append((t, float(parts[2]), float(parts[3]), parts[6:10]))
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
    pad = CLOCK_INTERVAL_MS / 1000.0
    inside = [r for r in rows if t0 - pad <= r[0] <= t1 + pad]
    window = "timed region"
    if not inside:
        mid = 0.5 * (t0 + t1)
        inside = [min(rows, key=lambda r: abs(r[0] - mid))]
        window = "nearest sample (timed region shorter than the sampling interval)"
    reasons = set()
    for _, _, _, flags in inside:
        for n, flag in zip(CLOCK_REASONS, flags):
            if flag.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(r[1] for r in inside),
            "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
            "samples": len(inside), "window": window,
            "region_ms": round(1000.0 * (t1 - t0), 1)}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons; only the samples taken while the
    timed region (begin() .. end()) runs are summarised."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"unstep_clocks_{os.getpid()}.csv")
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(CLOCK_INTERVAL_MS)],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:  # noqa: BLE001
            self.proc = None

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        time.sleep(2 * CLOCK_INTERVAL_MS / 1000.0)  # let a sample after the region land
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        t1 = self.t1 if self.t1 is not None else time.time()
        t0 = self.t0 if self.t0 is not None else t1
        return summarize_clocks(lines, t0, t1)


# ----------------------------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------------------------

def arm_config(wl, world, args):
    """The ``config`` object of a bench line, identical for the CUDA arm and the reference arm."""
    s = wl.shape
    Lk = wl.keys_for_chunk(wl.chunks - 1)
    fq = args.q_rope == "attn"
    strong = args.scaling == "strong"
    return {
        "workload": f"{wl.name}: B={s.B} H={s.H} D={s.D} grid={s.Hg}x{s.Wg} "
                    f"L={s.L} keys={Lk} window={wl.window} cap={wl.cap}",
        "per_rank": ("a (stream, head) shard of the workload, streams first, then heads"
                     if strong else "one independent copy of the workload per GPU")
        if world > 1 else "the whole workload",
        "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, then "
              f"{L2_FLUSH_BYTES >> 20} MiB read)",
        "parallelism": (f"(stream, head) shards x{world}" if strong else
                        f"independent streams x{world}"),
        "q_rope": "in the attention prologue (append moves k, v only)" if fq else
                  "in the append (q rotated in place)",
    }


def run_ours(args, rank, local_rank, world, emit=True):
    import torch
    from causal_video_diffusion_b200 import binding
    from causal_video_diffusion_b200 import workloads as W

    wl = W.WORKLOADS[args.workload]
    s = wl.shape
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    stream = torch.cuda.current_stream()
    last = wl.chunks - 1
    F = s.chunk_frames
    f_last = wl.frame_idx(last)
    Lk = wl.keys_for_chunk(last)
    strong = args.scaling == "strong" and world > 1
    if strong:
        # one workload split over the ranks: every rank draws the same activations and works on
        # its (stream, head) shard of them, in place; no collective touches the data
        from causal_video_diffusion_b200 import shard as S
        sh = S.plan(s.B, s.H, world)[rank]
        seed = args.seed
    else:
        # weak scaling: every rank streams its own copy of the workload (its own seed)
        sh = None
        seed = rank_seed(args.seed, rank)
    nb, nh = (sh.nb, sh.nh) if strong else (s.B, s.H)
    flops = wl.attn_flops(last)                          # the workload (one rank's, if weak)
    flops_rank = 4 * nb * nh * s.L * Lk * s.D            # what this rank's launches compute

    cache = binding.LayerCache(nb, nh, s.D, s.Hg, s.Wg, s.d_t, s.d_h, s.d_w,
                               cap_frames=wl.cap, max_pos_t=f_last + F, theta=s.theta,
                               shard=(sh.b0, sh.h0, s.B, s.H) if strong else None)
    # fill the cache: chunks 0 .. last-1, then the last chunk once
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device=dev)
    for c in range(wl.chunks):
        q, k, v = W.gen_qkv(W.qkv_seed(seed, chunk=c), s, device=str(dev))
        cache.rope_kv_append(q, k, v, wl.frame_idx(c), F)
        cache.window_attn(q, wl.window, out=out)
    q_src, k_src, v_src = W.gen_qkv(W.qkv_seed(seed, chunk=last, forward=1), s, device=str(dev))
    q_work = torch.empty_like(q_src)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer larger than L2, then read another one: L2 ends up holding clean lines
        # of neither the layer's inputs nor dirty data the next kernel would have to write back
        flush.zero_()
        flush_r.sum()
    torch.cuda.synchronize()
    if cache.device_error() != 0:
        raise RuntimeError("device error during cache fill")

    fq = args.q_rope == "attn"   # queries rotated inside the attention, not by the append

    def one_step(ev):
        q_work.copy_(q_src)
        flush_l2()                          # evict L2 between timed steps
        ev[0].record(stream)
        # re-forward of the last chunk
        cache.rope_kv_append(q_work, k_src, v_src, f_last, F, defer_q=fq)
        ev[1].record(stream)
        cache.window_attn(q_work, wl.window, out=out, rope_q=fq)
        ev[2].record(stream)

    for _ in range(args.warmup):
        one_step([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler.begin()
    for i in range(args.steps):
        one_step(events[i])
    torch.cuda.synchronize()
    sampler.end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    rope_ms = [e[0].elapsed_time(e[1]) for e in events]
    attn_ms = [e[1].elapsed_time(e[2]) for e in events]
    step_ms_local = sum(r + a for r, a in zip(rope_ms, attn_ms)) / args.steps
    step_ms = reduce_max(step_ms_local, world, dev)
    err = cache.device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} in the timed region")

    # e2e through the public API from pinned host buffers: every step copies its q, k, v in
    # and its output out; the pipeline overlaps step i's copies with step i-1's compute
    q_h = q_src.cpu().pin_memory()
    k_h = k_src.cpu().pin_memory()
    v_h = v_src.cpu().pin_memory()
    out_h = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16).pin_memory()
    pipe = binding.HostStepPipeline(cache, rope_q_in_attn=fq)
    e2e_steps = max(4, min(args.steps, 100))
    pipe.run(q_h, k_h, v_h, f_last, F, wl.window, out_h, 4)            # warm-up
    e2e_ms = reduce_max(pipe.run(q_h, k_h, v_h, f_last, F, wl.window, out_h, e2e_steps)
                        / e2e_steps, world, dev)
    if cache.device_error() != 0:
        raise RuntimeError("device error in the e2e region")

    peaks, peak_src = load_peaks()
    attn_avg = reduce_max(sum(attn_ms) / args.steps, world, dev)
    rope_avg = reduce_max(sum(rope_ms) / args.steps, world, dev)
    attn_tflops = flops_rank / (attn_avg * 1e-3) / 1e12
    rope_bytes = wl.rope_bytes(rotate_q=not fq) * nb * nh // (s.B * s.H)
    rope_gbs = rope_bytes / (rope_avg * 1e-3) / 1e9
    job_flops = flops if strong else world * flops     # all ranks together
    value = job_flops / (step_ms * 1e-3) / 1e12
    e2e_value = job_flops / (e2e_ms * 1e-3) / 1e12
    act_bytes = s.B * s.L * s.H * s.D * 2
    rope_traffic = profile_traffic(f"rope_kv_append_{wl.name}.txt", ROPE_SOURCES)
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "strong" if strong else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) fp32 draws rounded to bf16 (q, k, v)",
        "config": arm_config(wl, world, args),
        "chunk_steps_per_s": round((1 if strong else world) * s.B / (step_ms * 1e-3), 2),
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "h2d_bytes_per_step": 3 * act_bytes, "d2h_bytes_per_step": act_bytes,
                "how": "pinned host q/k/v -> device, both calls, device -> pinned host out, "
                       "every step; copies of neighbouring steps overlap the compute; steps back "
                       "to back (working set > L2)"},
        "gpu_launches": 2 * args.steps,
        "gpu_launches_e2e": 2 * e2e_steps,
        "roofline": {
            "kernel": f"window_attn_kernel<{s.D}, {str(fq).lower()}>",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": peaks["bf16_tflops"],
            "peak_source": f"{peak_src} bf16 burst",
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / peaks["bf16_tflops"], 4),
            "traffic": profiled_traffic(wl.name, rope_q=fq),
            "ms_per_launch": round(attn_avg, 4),
            "flops_per_launch": flops_rank,
        },
        "rope_roofline": {
            "kernel": f"rope_kv_append_kernel<{s.D}, {str(not fq).lower()}>",
            "bound": "hbm",
            "achieved": round(rope_gbs, 1),
            "peak": peaks["hbm_gbs"],
            "peak_source": f"{peak_src} copy",
            "unit": "GB/s",
            "frac": round(rope_gbs / peaks["hbm_gbs"], 4),
            "bytes_per_launch": rope_bytes,
            "us_per_launch": round(rope_avg * 1e3, 2),
            # DRAM bytes of one launch from the committed ncu capture, and the rate DRAM itself
            # sees during the launch (the cache writes mostly stay in L2 until later kernels)
            "traffic": rope_traffic,
            "dram_gbs": None if rope_traffic is None else
            round(rope_traffic / (rope_avg * 1e-3) / 1e9, 1),
        },
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, q_src, k_src, v_src, cache, args)
    if (rank == 0 and world == 1 and emit and args.workload == "wan_full"
            and not args.no_other_workloads):
        del cache, q_src, k_src, v_src, out
        try:
            result["other_workloads"] = other_workloads(args, local_rank)
        except Exception as e:  # noqa: BLE001 -- the headline line is printed regardless
            result["other_workloads"] = {"error": f"{type(e).__name__}: {str(e)[:200]}"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and emit:
        print(json.dumps(result), flush=True)
    return result


# ----------------------------------------------------------------------------------------------
# the oracle on the host cores
# ----------------------------------------------------------------------------------------------

def _oracle_sample(wl, q_bits, k_bits, v_bits, heads, rows_per_head, seed=0):
    """Time the oracle on a bounded sample of one step: the heads in ``heads`` (RoPE of their q
    and k over the whole chunk, appended to a cache streamed to the last chunk) and attention for
    ``rows_per_head`` query rows of each.  Heads are independent and rows cost the same, so the
    step's time is extrapolated by H/len(heads) for the RoPE and by rows for the attention.
    Returns (extrapolated step seconds, measured seconds, sample description)."""
    import numpy as np
    import oracle
    s = wl.shape
    hs = list(heads)
    qs, ks, vs = (np.ascontiguousarray(a[:, :, hs, :]) for a in (q_bits, k_bits, v_bits))
    ol = oracle.OracleLayer(s.B, len(hs), s.Hg, s.Wg,
                            oracle.RopeSpec(s.d_t, s.d_h, s.d_w, s.theta), wl.cap)
    last = wl.chunks - 1
    for c in range(last):
        ol.fill_zero_frames(wl.frame_idx(c), s.chunk_frames)
    t0 = time.perf_counter()
    q_rot = ol.append(qs, ks, vs, wl.frame_idx(last), s.chunk_frames)
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    rows = [(b, int(l), h) for b in range(s.B) for h in range(len(hs))
            for l in rng.choice(s.L, size=min(rows_per_head, s.L), replace=False)]
    t2 = time.perf_counter()
    ol.attend(q_rot, wl.window, rows)
    t3 = time.perf_counter()
    total_rows = s.B * s.H * s.L
    step_s = (t1 - t0) * s.H / len(hs) + (t3 - t2) * total_rows / len(rows)
    sample = (f"RoPE+append of {len(hs)} of {s.H} heads over the whole chunk and fp64 attention "
              f"of {len(rows)} of {total_rows} query rows, extrapolated to one full step")
    return step_s, (t1 - t0) + (t3 - t2), sample


def cpu_baseline(wl, q, k, v, cache, args):
    import oracle
    from causal_video_diffusion_b200 import workloads as W
    cores = len(os.sched_getaffinity(0))
    oracle.set_num_threads(cores)
    qb, kb, vb = (W.bits(t.cpu()) for t in (q, k, v))
    H = wl.shape.H
    heads = sorted({0, H // 3, (2 * H) // 3, H - 1})   # four heads at the shape benchmarked
    step_s, measured, sample = _oracle_sample(wl, qb, kb, vb, heads, args.cpu_rows)
    used = oracle.num_threads()
    flops = wl.attn_flops(wl.chunks - 1)
    # the same oracle on one thread, on a smaller sample of the same step
    oracle.set_num_threads(1)
    step1_s, measured1, sample1 = _oracle_sample(wl, qb, kb, vb, [0], max(1, args.cpu_rows // 64))
    oracle.set_num_threads(cores)
    return {"value": round(flops / step_s / 1e12, 6), "unit": "TFLOP/s",
            "cores": used, "kind": "oracle", "sample": sample,
            "seconds_measured": round(measured, 3), "extrapolated_step_s": round(step_s, 3),
            "value_1thread": round(flops / step1_s / 1e12, 6), "sample_1thread": sample1,
            "seconds_measured_1thread": round(measured1, 3)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from causal_video_diffusion_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    s = wl.shape
    cores = len(os.sched_getaffinity(0))
    oracle.set_num_threads(cores)
    q, k, v = W.gen_qkv(W.qkv_seed(args.seed, chunk=wl.chunks - 1, forward=1), s)
    qb, kb, vb = W.bits(q), W.bits(k), W.bits(v)
    for i in range(args.warmup):
        _oracle_sample(wl, qb, kb, vb, [i % s.H], args.ref_rows, seed=i)
    total = 0.0
    measured = 0.0
    sample = ""
    for i in range(args.steps):
        step_s, meas_s, sample = _oracle_sample(wl, qb, kb, vb, [i % s.H], args.ref_rows,
                                                seed=i)
        total += step_s
        measured += meas_s
    step_s = total / args.steps
    flops = wl.attn_flops(wl.chunks - 1)
    value = flops / step_s / 1e12
    result = {
        "metric": METRIC, "impl": "reference", "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # a full step of the fp64 oracle takes minutes: every step runs a bounded sample and
        # its time is scaled up to the whole step; ms_per_step is that extrapolated figure and
        # seconds_measured the wall time the timed samples actually took
        "ms_per_step": round(step_s * 1e3, 3), "extrapolated": True,
        "seconds_measured": round(measured, 3),
        "ms_per_step_measured": round(measured / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "strong" if args.scaling == "strong" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic: seeded N(0,1) bf16",
        "config": arm_config(wl, world, args),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": "per step: " + sample + " (extrapolated)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def run_lowrank(args, rank, local_rank, world, emit=True):
    """The truncated-SVD V and O projections of one chunk (4680 tokens, 1536 -> rank 1413
    stored padded to 1472 -> 1536): four tensor-core GEMMs per step."""
    import torch
    from causal_video_diffusion_b200 import binding
    from causal_video_diffusion_b200 import lowrank
    from causal_video_diffusion_b200 import workloads as W
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    d, M = W.MODEL_DIM, W.WORKLOADS["wan_full"].shape.L
    r = lowrank.padded(lowrank.retained_rank(d))
    facs = [tuple(t.to(dev) for t in lowrank.svd_factors(W.gen_weight(args.seed + i, d, d),
                                                          lowrank.retained_rank(d)))
            for i in range(2)]
    x = W.gen_act(args.seed + 7, M, d, device=str(dev))
    tb = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    yv = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
    yo = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev):
        flush.zero_()
        flush_r.sum()
        ev[0].record(stream)
        binding.lowrank_linear(x, facs[0][0], facs[0][1], t=tb, y=yv, dev_error=err)
        binding.lowrank_linear(yv, facs[1][0], facs[1][1], t=tb, y=yo, dev_error=err)
        ev[1].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler.begin()
    for e in evs:
        step(e)
    torch.cuda.synchronize()
    sampler.end()
    clocks = sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError("device error in the projections")
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    # FLOPs on the retained rank (1413): the zero padding of the factors is not counted as work
    flops = 2 * (2 * M * d * lowrank.retained_rank(d) * 2)
    peaks, src = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    result = {
        "metric": "truncated-SVD V/O projection TFLOP/s at Wan-1.3B shape (rank 0.92)",
        "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic N(0,1/d) weights and N(0,1) activations",
        "config": {"workload": f"lowrank_vo: M={M} d={d} rank={lowrank.retained_rank(d)} "
                               f"(stored padded to {r}), V then O",
                   "l2": "flushed between steps"},
        "scaling": "weak", "vs_baseline": None,
        "gpu_launches": 4 * args.steps,
        "roofline": {"kernel": "gemm2sm_bf16_tn_kernel (CTA pairs)", "bound": "tensor",
                     "achieved": round(tf, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4), "peak_source": src,
                     "traffic": profile_traffic("gemm_bf16_lowrank_vo.txt", GEMM_SOURCES)},
        "clocks": clocks,
        "cpu_baseline": None if args.no_cpu_baseline else
        _lowrank_cpu_baseline(x, facs, flops, M)}
    if emit:
        print(json.dumps(result), flush=True)
    return result


def _lowrank_cpu_baseline(x, facs, flops, M, rows=None):
    """The fp64 oracle of the same four products on ``rows`` tokens (default all M),
    extrapolated to M."""
    import oracle
    from causal_video_diffusion_b200 import workloads as W
    rows = M if rows is None else rows
    xb = W.bits(x[:rows].cpu())
    (a1, a2), (b1, b2) = [(W.bits(f1.cpu()), W.bits(f2.cpu())) for f1, f2 in facs]
    t0 = time.perf_counter()
    yv = oracle.lowrank_linear(xb, a1, a2)
    oracle.lowrank_linear(oracle.f64_to_bf16(yv), b1, b2)
    dt = time.perf_counter() - t0
    step_s = dt * M / rows
    return {"value": round(flops / step_s / 1e12, 6), "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"the V and O projections of {rows} of {M} tokens in fp64 (numpy)"
                      + (", extrapolated to the whole step" if rows < M else ""),
            "seconds_measured": round(dt, 3)}


def run_vae_conv(args, rank, local_rank, world, emit=True):
    """The VAE decoder's causal 3x3x3 convolution at the latent resolution: one 3-frame chunk of
    the 60x104 latent with its 2 history frames, 384 -> 384 channels (channels-last bf16)."""
    import numpy as np
    import torch
    from causal_video_diffusion_b200 import binding
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, T, H, Wd, C = 1, 3, 60, 104, 384
    g = torch.Generator(device=dev)
    g.manual_seed(args.seed)
    x = torch.randn((B, T + 2, H, Wd, C), generator=g, device=dev).to(torch.bfloat16)
    w = (torch.randn((C, 3, 3, 3, C), generator=g, device=dev) / np.sqrt(27 * C)).to(torch.bfloat16)
    bias = torch.randn((C,), generator=g, device=dev, dtype=torch.float32) * 0.1
    y = torch.empty((B, T, H, Wd, C), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    scratch = binding.conv3d_scratch(dev)   # stream-K tail over the SMs
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev):
        flush.zero_()
        flush_r.sum()
        ev[0].record(stream)
        binding.conv3d_causal(x, w, bias, out=y, dev_error=err, scratch=scratch)
        ev[1].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler.begin()
    for e in evs:
        step(e)
    torch.cuda.synchronize()
    sampler.end()
    clocks = sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError("device error in the convolution")
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    flops = 2 * B * T * H * Wd * C * 27 * C
    peaks, src = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    result = {
        "metric": "VAE decoder causal 3x3x3 conv TFLOP/s at the 60x104 latent (384 -> 384)",
        "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic N(0,1) activations, N(0,1/(27 C)) weights",
        "config": {"workload": f"vae_conv: B={B} T={T}(+2 history) H={H} W={Wd} C_in={C} "
                               f"C_out={C}, channels-last", "l2": "flushed between steps"},
        "scaling": "weak", "vs_baseline": None,
        "gpu_launches": args.steps,
        "roofline": {"kernel": "conv3d_causal_pair_kernel", "bound": "tensor", "achieved": round(tf, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4), "peak_source": src,
                     "flops_per_launch": flops,
                     "traffic": profile_traffic("conv3d_vae_conv.txt", CONV_SOURCES)},
        "clocks": clocks,
        "cpu_baseline": None if args.no_cpu_baseline else
        _conv_cpu_baseline(x, w, bias, flops, H)}
    if emit:
        print(json.dumps(result), flush=True)
    return result


def _conv_cpu_baseline(x, w, bias, flops, H, rows=None):
    """The fp64 oracle of the same layer on a band of ``rows`` output rows (default all H),
    extrapolated."""
    import oracle
    from causal_video_diffusion_b200 import workloads as W
    rows = H if rows is None else rows
    xb = W.bits(x[:, :, :rows].cpu())
    wb = W.bits(w.cpu())
    t0 = time.perf_counter()
    oracle.conv3d_causal(xb, wb, bias.double().cpu().numpy())
    dt = time.perf_counter() - t0
    step_s = dt * H / rows
    return {"value": round(flops / step_s / 1e12, 6), "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{rows} of {H} output rows of every frame and channel in fp64 (numpy)"
                      + (", extrapolated to the whole layer" if rows < H else ""),
            "seconds_measured": round(dt, 3)}


def run_clip(args, rank, local_rank, world, emit=True):
    """The 5-s clip through 30 attention layers (Table 3 schedule: 23 forwards), eagerly and as
    one CUDA graph; inputs of all 690 calls pre-generated on the device."""
    import torch
    from causal_video_diffusion_b200 import clip
    from causal_video_diffusion_b200 import workloads as W
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS["clip30"]
    drv = clip.ClipDriver(wl, seed=args.seed, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    drv.run()                                  # warm-up (first calls set kernel attributes)
    torch.cuda.synchronize()
    drv.reset()
    e0, e1 = ev(), ev()
    e0.record()
    drv.run()
    e1.record()
    e1.synchronize()
    eager_ms = e0.elapsed_time(e1)
    drv.reset()
    drv.capture()
    for _ in range(max(1, args.warmup // 3)):
        drv.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    reps = max(1, min(args.steps, 10))
    e0, e1 = ev(), ev()
    sampler.begin()
    e0.record()
    for _ in range(reps):
        drv.replay()
    e1.record()
    e1.synchronize()
    sampler.end()
    clocks = sampler.stop()
    graph_ms = e0.elapsed_time(e1) / reps
    for c in drv.caches:
        if c.device_error() != 0:
            raise RuntimeError("device error in the clip")
    flops = drv.attn_flops()
    peaks, src = load_peaks()
    tf = flops / (graph_ms * 1e-3) / 1e12
    result = {
        "metric": "attention-layer TFLOP/s over a 5-s clip (30 layers x 23 forwards)",
        "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": reps,
        "warmup": args.warmup, "ms_per_step": round(graph_ms, 3), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic seeded N(0,1) bf16 q/k/v per (forward, layer)",
        "config": {"workload": "clip30: 7 chunks x (5,3,3,3,3,3,3) forwards x 30 layers, W=9",
                   "calls": drv.calls, "graph": "one CUDA graph per clip"},
        "eager_ms_per_clip": round(eager_ms, 3),
        "chunk_steps_per_s": round(drv.calls / (graph_ms * 1e-3), 1),
        "attention_only_frames_per_s": round(81 / (graph_ms * 1e-3), 1),
        "scaling": "weak", "vs_baseline": None,
        "gpu_launches": (2 * drv.layers + 1) * len(drv.sched),
        "roofline": {"kernel": "window_attn_kernel<128, false> (with the RoPE+append and renoise "
                               "launches of every forward)", "bound": "tensor",
                     "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4), "peak_source": src,
                     "traffic": None},
        "frac_of_peak": round(tf / peaks["bf16_tflops"], 4), "clocks": clocks}
    del drv
    if emit:
        print(json.dumps(result), flush=True)
    return result


OTHER_WORKLOADS = ("wan_window", "long_b4", "clip30", "lowrank_vo", "vae_conv")


def other_workloads(args, local_rank):
    """The other layer configurations and the measured "next" rows, timed in the same process
    after the full-cache line (20 steps each after 5 warm-up steps, L2 flushed between steps, no
    CPU baseline; the clip: 3 graph replays after an eager run and one replay), summarised for the
    default bench line."""
    import torch
    out = {}
    for name in OTHER_WORKLOADS:
        a = argparse.Namespace(**vars(args))
        a.workload, a.steps, a.warmup, a.no_cpu_baseline = name, 20, 5, True
        a.no_other_workloads = True
        try:
            if name == "lowrank_vo":
                r = run_lowrank(a, 0, local_rank, 1, emit=False)
            elif name == "clip30":
                a.steps, a.warmup = 3, 3   # one graph replay per clip: 3 timed after 1
                r = run_clip(a, 0, local_rank, 1, emit=False)
            elif name == "vae_conv":
                r = run_vae_conv(a, 0, local_rank, 1, emit=False)
            else:
                r = run_ours(a, 0, local_rank, 1, emit=False)
        except Exception as e:  # noqa: BLE001 -- the headline line is printed regardless
            out[name] = {"error": f"{type(e).__name__}: {str(e)[:200]}"}
            continue
        entry = {"workload": r["config"]["workload"], "value": r["value"], "unit": r["unit"],
                 "ms_per_step": r["ms_per_step"], "steps": r["steps"],
                 "roofline_frac": r["roofline"]["frac"], "roofline_kernel": r["roofline"]["kernel"],
                 "traffic": r["roofline"].get("traffic"),
                 "clocks": {k: r["clocks"].get(k) for k in ("sm_mhz", "reasons", "samples")}}
        if "rope_roofline" in r:
            entry["rope_gbs"] = r["rope_roofline"]["achieved"]
            entry["rope_frac"] = r["rope_roofline"]["frac"]
        if "chunk_steps_per_s" in r:
            entry["chunk_steps_per_s"] = r["chunk_steps_per_s"]
        if "eager_ms_per_clip" in r:
            entry["eager_ms_per_clip"] = r["eager_ms_per_clip"]
        out[name] = entry
        torch.cuda.empty_cache()
    return out


def launch_ranks(n: int, argv, port: int = 0) -> int:
    """Run this script as ``n`` ranks under torch.distributed.run on 127.0.0.1 (one process
    per GPU), bounded by a timeout; returns the launcher's exit status."""
    import socket
    if port == 0:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
    cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan_full",
                    help="wan_full (default), wan_window, long_b4, wan_full_h8, tiny; or the "
                         "separate legs lowrank_vo, clip30, vae_conv")
    ap.add_argument("--seed", type=int, default=2024)
    ap.add_argument("--cpu-rows", type=int, default=8192,
                    help="oracle rows per head (at most the chunk's queries) of the CPU baseline")
    ap.add_argument("--ref-rows", type=int, default=32, help="oracle rows per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the other workloads' summary that the default full-cache line "
                         "carries at N = 1")
    ap.add_argument("--q-rope", choices=["append", "attn"], default="append",
                    help="where the queries are rotated: in the append (q in place) or in the "
                         "attention's prologue")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: every GPU streams its own copy of the workload; strong: the "
                         "workload's (stream, head) grid is split over the GPUs, streams first")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started without a launcher: start one rank per GPU and pass on their exit status
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    rank, local_rank, world = dist_env()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "lowrank_vo":
        run_lowrank(args, rank, local_rank, world)
    elif args.workload == "clip30":
        run_clip(args, rank, local_rank, world)
    elif args.workload == "vae_conv":
        run_vae_conv(args, rank, local_rank, world)
    else:
        run_ours(args, rank, local_rank, world)


if __name__ == "__main__":
    main()
