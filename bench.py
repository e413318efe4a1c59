"""Steady-state throughput of the FIFO denoising queue on B200 (one JSON line).

A step is one dp_queue_step over a full queue (every level occupied: one
batched DiT pass over all queued chunks, the Euler update in the ring, the
push of a fresh N(0,1) chunk) plus the dp_queue_pop of the clean chunk.
Workload: the Wan2.1-1.3B-shaped random-init model (30 layers, dim 1536,
12 heads, FFN 8960), 480x832 video -> 16-ch 60x104 latent, chunks of 2 latent
frames (3120 tokens), T = 50 levels, 512 prompt tokens.  Metric: latent
frames/s (2 frames leave the queue per step) and the fraction of the bf16
tensor-core peak reached by the step's algorithmic FLOPs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--fill steps|load] [--plateau]
                    [--neighbours pred|both] [--qk-norm-rope]
    python bench.py --stream [--workload wan1.3b_480p_long] [--stream-lengths 32,64]

N > 1 runs N independent replicas (one queue per GPU, no collective on the
data path), launched by torch.distributed.run.  --impl reference times the
float64 CPU oracle on a bounded sample of the same step (rank 0 only).
--fill load places the steady state with dp_queue_load_state instead of T-1
real steps (needed for the Wan-14B shapes, where a step takes seconds);
--plateau also times the partial-queue steady state of a stream shorter than
the queue.  Besides the metric, the line reports the roofline of the GEMM
class, the per-class kernel times (from a separate instrumented pass),
end-to-end throughput with host buffers (host clock), clocks sampled during
the timed region, device memory and the CPU oracle.
--stream runs whole streams instead (every step from the first push to the
last pop, popping to host), for the workload's own length and the lengths of
--stream-lengths, and reports the steady-state and whole-stream rates and the
peak device memory of each, which does not depend on the stream length.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "latent frames/s per B200 (steady-state queue); % of bf16 tensor-core peak"
UNIT = "latent frames/s"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK)
    d["_source"] = "fallback"
    return d


def gemm_traffic():
    """DRAM bytes per gemm_tc_kernel launch from the committed ncu launch list,
    or None when the kernel source changed since the counters were taken."""
    import hashlib
    import re
    src = os.path.join(ROOT, "chunked_fifo_denoising_b200", "csrc")
    h = hashlib.sha256()
    for f in ("k_gemm_tc.cu", "tc_common.cuh"):
        with open(os.path.join(src, f), "rb") as fh:
            h.update(fh.read())
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_traffic_wan1.3b.md")) as fh:
            text = fh.read()
    except OSError:
        return None
    m = re.search(r"traffic gemm_tc_kernel bytes_per_launch=(\d+) source_sha256_16=([0-9a-f]+)", text)
    if not m or m.group(2) != h.hexdigest()[:16]:
        return None
    return int(m.group(1))


def step_flops(m, q, occ, neighbours="pred"):
    """Algorithmic FLOPs of one step with `occ` queued chunks, every chunk with
    a full predecessor: per token per layer 12 d^2 + 4 d F + 4 (2 Lc) d + 4 Lt d,
    plus the patch and head projections (2 * 64 * d each per token).  With the
    successor link, every chunk but the last also reads Lc more keys."""
    Lc = q.tokens_per_chunk(m)
    d, F = m.dim, m.ffn_dim
    per_tok_layer = 12 * d * d + 4 * d * F + 4 * (2 * Lc) * d + 4 * m.text_len * d
    toks = occ * Lc
    flops = toks * (m.n_layers * per_tok_layer + 2 * 2 * m.patch_dim * d)
    if neighbours == "both":
        flops += m.n_layers * 4.0 * Lc * ((occ - 1) * Lc) * d
    return flops


class Clocks:
    """Samples nvidia-smi clocks and throttle reasons while alive."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = str(index)
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.f.read().splitlines():
            c = [x.strip() for x in ln.split(",")]
            if len(c) < 9 or c[0] != self.index:
                continue
            try:
                sm.append(float(c[1]))
                mx = max(mx, float(c[2]))
            except ValueError:
                continue
            for n, v in zip(names, c[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def visible_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",")]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------------------
# CPU oracle sample
# ---------------------------------------------------------------------------

_ORACLE_CASE = {}


def _oracle_case(w):
    """Inputs of the CPU sample, built once (parameter generation is untimed)."""
    if w.name not in _ORACLE_CASE:
        import numpy as np

        import synth
        from oracle import dit

        m1 = synth.truncated(w, 1).model
        q = w.queue
        p = synth.make_params(m1)
        text = synth.make_text(m1)
        fn = dit.make_velocity_fn(p, text, m1, q.T)   # prompt K/V: once per prompt, untimed
        lat = synth.make_noise(m1, q, 0).astype(np.float64)
        rng = np.random.default_rng(0)
        Lc = q.tokens_per_chunk(m1)
        kv = [(rng.standard_normal((Lc, m1.dim)) * 0.5, rng.standard_normal((Lc, m1.dim)) * 0.5)]
        _ORACLE_CASE[w.name] = (fn, lat, kv)
    return _ORACLE_CASE[w.name]


def oracle_sample(w, reps=1):
    """Times the oracle on one chunk through one layer of the step (with its
    predecessor K/V) and scales to a full steady-state step.  Returns
    (frames/s extrapolated, seconds per sample, threads)."""
    q = w.queue
    fn, lat, kv = _oracle_case(w)
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        fn([lat], [q.T // 2], [5], kv, None)
        times.append(time.perf_counter() - t0)
    t = min(times)
    per_step = t * q.T * w.model.n_layers      # every queued chunk, every layer
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    return q.frames_per_chunk / per_step, t, threads


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank values (every rank gets the result)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def measure_plateau(model, m, q, text, occ, steps, warmup, g, dist, world, rank, peak_tf):
    """A stream shorter than the queue never fills it: from the push of its
    last chunk until its first chunk pops, `occ` chunks advance one level per
    step with no push and no pop.  Places that state (chunks 0 .. occ-1 at
    levels T-occ .. T-1, chunk 0 without a predecessor) and times `steps`
    plateau steps.  A chunk needs T steps, so the stream's rate is
    occ / T chunks per step."""
    import torch

    from chunked_fifo_denoising_b200 import Queue
    T = q.T
    if warmup + steps > T - occ:
        raise SystemExit(f"plateau of {T - occ} steps is shorter than warm-up + steps")
    queue = Queue(model, text, T, q.frames_per_chunk, q.lat_h, q.lat_w, occ, ready_capacity=2,
                  seed=3 + rank)
    lat = torch.randn((occ,) + queue.chunk_shape, generator=g, device="cuda")
    queue.load_state(occ, occ, lat)
    del lat
    info = queue.inspect()
    assert info["n"] == occ and info["head_pred"] == 0 and info["levels"][0] == T - occ, info
    for _ in range(warmup):
        queue.step(None)
    queue.sync()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        queue.step(None)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1)], dist, device="cuda")[0]
    queue.sync()
    queue.close()
    Lc = q.tokens_per_chunk(m)
    flops = step_flops(m, q, occ) - m.n_layers * 4.0 * Lc * Lc * m.dim  # chunk 0: own keys only
    step_s = ms / steps / 1e3
    return {"occupancy": occ, "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
            "value": world * occ * q.frames_per_chunk / T / step_s, "unit": UNIT,
            "step_tflop": flops / 1e12, "pct_bf16_peak": 100.0 * flops / step_s / (peak_tf * 1e12)}


def whole_job_rate(world, steps, frames_per_step, ms):
    """Units of all ranks (weak scaling: each rank runs its own replica) over
    the slowest rank's time."""
    return world * steps * frames_per_step / (ms / 1e3)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals = []
    t_sample = 0.0
    threads = 1
    t_start = time.perf_counter()
    for i in range(args.warmup + args.steps):
        v, t_sample, threads = oracle_sample(w)
        if i >= args.warmup:
            vals.append(v)
    v = statistics.median(vals)
    scale = w.queue.T * w.model.n_layers
    sample = (f"1 chunk x 1 layer of the {w.name} step (with its predecessor K/V), "
              f"{t_sample:.1f} s each, scaled by T x layers = {scale}")
    # Each timed "step" is one bounded sample: ms_per_step is the extrapolated
    # time of a whole step, not the time this run spent per sample.
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.queue.frames_per_chunk / v * 1e3,
            "extrapolated": True,
            "measured": {"samples": args.steps, "warmup_samples": args.warmup,
                         "seconds_per_sample": t_sample, "sample_scale_to_step": scale,
                         "wall_s": time.perf_counter() - t_start},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def setup_rank():
    """(world, rank, local rank, torch.distributed or None) of this process."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    return world, rank, local, dist


def build_model(m, g, stream, neighbours):
    """The model with random-init weights drawn on the device, N(0, 0.02^2)
    (RMSNorm weights around 1), and a N(0,1) prompt."""
    import torch

    import synth
    from chunked_fifo_denoising_b200 import Model
    model = Model(m, "bf16", stream=stream, neighbours=neighbours)
    for name, shape, per_layer in synth.param_specs(m):
        for l in range(m.n_layers if per_layer else 1):
            t = torch.randn(shape, generator=g, device="cuda") * 0.02
            if name.endswith("norm.w"):
                t += 1.0
            model.set_param(name, t, l)
            del t
    text = torch.randn((m.text_len, m.text_in_dim), generator=g, device="cuda")
    return model, text


def run_ours(args, w):
    import torch

    from chunked_fifo_denoising_b200 import Queue

    world, rank, local, dist = setup_rank()
    if args.qk_norm_rope:
        import synth as _s
        w = _s.with_qk_norm_rope(w)
    m, q = w.model, w.queue
    T = q.T
    occ = T
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cuda").manual_seed(1000 + rank)   # seeded per rank
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    model, text = build_model(m, g, stream, args.neighbours)
    n_chunks = T + 1 + args.warmup + args.steps + args.kernel_steps + args.e2e_steps + 2
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    queue = Queue(model, text, T, q.frames_per_chunk, q.lat_h, q.lat_w, n_chunks,
                  ready_capacity=2, seed=3 + rank)
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info()[0]
    out = torch.empty(queue.chunk_shape, device="cuda")
    if args.fill == "steps":
        # T-1 real steps bring the queue to full occupancy (untimed)
        for _ in range(T - 1):
            queue.step(None)
            queue.try_pop(out)
    else:
        # the steady state placed directly: chunks 1..T-1 at levels 1..T-1 (the
        # step pushes chunk T at level T), and the persisted K/V of chunk 0
        # (popped last step) for the head's predecessor
        lat = torch.randn((T - 1,) + queue.chunk_shape, generator=g, device="cuda")
        kv = torch.randn((m.n_layers, 2, queue.tokens, m.dim), generator=g, device="cuda")
        queue.load_state(T, T, lat, kv)
        del lat, kv
    queue.sync()
    info = queue.inspect()
    assert info["n"] == occ, info
    # placed state: the head reads its predecessor's persisted K/V (after a real
    # fill the first warm-up step's head is chunk 0, which has none)
    assert args.fill == "steps" or info["head_pred"] != 0, info
    for _ in range(args.warmup):
        queue.step(None)
        queue.pop(out)
    queue.sync()
    # timed region: K full steps (no per-kernel instrumentation inside it)
    clocks = Clocks(visible_index(local))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        queue.step(None)
        queue.pop(out)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ck = clocks.stop()
    queue.sync()
    ms = e0.elapsed_time(e1)
    # per-kernel breakdown from a separate instrumented pass (CUDA events
    # around every launch on the queue's stream)
    queue.set_timing(True)
    torch.cuda.synchronize()
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    for _ in range(args.kernel_steps):
        queue.step(None)
        queue.pop(out)
    k1.record(stream)
    torch.cuda.synchronize()
    ms_instr = k0.elapsed_time(k1)
    kt = queue.timing()
    queue.set_timing(False)
    queue.sync()
    # end to end through the public API with page-locked host buffers: every
    # step copies its noise chunk in (H2D) and the popped chunk out (D2H, the
    # call returns once it has landed); host clock around the calls
    hn = torch.randn(queue.chunk_shape, generator=torch.Generator().manual_seed(rank)).pin_memory()
    ho = torch.empty(queue.chunk_shape).pin_memory()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.e2e_steps):
        queue.step(hn)
        queue.pop(ho)
    torch.cuda.synchronize()
    ms_e2e = (time.perf_counter() - t0) * 1e3
    queue.sync()
    # max over ranks
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], dist, device="cuda")
    frames = q.frames_per_chunk
    value = whole_job_rate(world, args.steps, frames, ms)
    e2e_value = whole_job_rate(world, args.e2e_steps, frames, ms_e2e)
    pk = peaks()
    flops = step_flops(m, q, occ, args.neighbours)
    ms_step = ms / args.steps
    peak_tf = pk["bf16_tflops_sustained"]
    gemm = kt["gemm"]
    attn = kt["self_attention"]
    ks = args.kernel_steps
    # launches of the library's kernels per step (counted by its per-class timer)
    launches_per_step = sum(v["launches"] for v in kt.values()) / ks
    roof = {"bound": "tensor", "kernel": "gemm_tc (tcgen05 GEMM, all fused epilogues)",
            "achieved": gemm["flops"] / (gemm["ms"] / 1e3) / 1e12 if gemm["ms"] > 0 else None,
            "peak": peak_tf, "unit": "TFLOP/s",
            "peak_source": f"{pk['_source']} bf16_tflops_sustained (kernel timed inside a long step)",
            "traffic": gemm_traffic(),
            "traffic_unit": "bytes per launch (ncu, small per-kernel captures scaled to full size; mean of the six GEMM shapes)"}
    if roof["achieved"]:
        roof["frac"] = roof["achieved"] / peak_tf
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) noise and prompt, N(0,0.02^2) random-init weights",
            "config": {"workload": w.name, "T": T, "occupancy": occ, "chunk_tokens": q.tokens_per_chunk(m),
                       "tokens_per_step": occ * q.tokens_per_chunk(m), "frames_per_step": frames,
                       "layers": m.n_layers, "dim": m.dim, "ffn": m.ffn_dim, "heads": m.n_heads,
                       "text_tokens": m.text_len, "neighbours": args.neighbours,
                       "qk_norm_rope": bool(args.qk_norm_rope),
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (fp32 residual stream alone is "
                             f"{occ * q.tokens_per_chunk(m) * m.dim * 4 / 1e6:.0f} MB)"},
            "pct_bf16_peak": 100.0 * flops / (ms_step / 1e3) / (peak_tf * 1e12),
            "step_tflop": flops / 1e12,
            "roofline": roof,
            "kernels": {k: {"ms_per_step": v["ms"] / ks, "launches_per_step": v["launches"] / ks,
                            "tflops": (v["flops"] / (v["ms"] / 1e3) / 1e12) if v["ms"] > 0 and v["flops"] else None,
                            "gbs": (v["bytes"] / (v["ms"] / 1e3) / 1e9) if v["ms"] > 0 and v["bytes"] else None}
                        for k, v in kt.items() if v["launches"]},
            "kernels_pass": {"steps": ks, "ms_per_step_instrumented": ms_instr / ks,
                             "note": "separate pass after the timed region, CUDA events around every launch"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(hn.numel() * 4),
                    "d2h_bytes_per_step": int(ho.numel() * 4), "steps": args.e2e_steps,
                    "clock": "host perf_counter around dp_queue_step(host noise) + dp_queue_pop(host out)"},
            "gpu_launches": int(round(launches_per_step * args.steps)), "clocks": ck,
            "memory": {"model_bytes": int(free0 - free1), "queue_bytes": int(free1 - free2),
                       "source": "cudaMemGetInfo around dp_model_create+set_param and dp_queue_init"},
            "fill": args.fill}
    if attn["ms"] > 0:
        line["self_attention_tflops"] = attn["flops"] / (attn["ms"] / 1e3) / 1e12
    if args.plateau:
        if 0 < q.n_chunks < T:
            queue.close()
            line["plateau"] = measure_plateau(model, m, q, text, q.n_chunks, args.steps, args.warmup, g,
                                              dist, world, rank, peak_tf)
        else:
            line["plateau"] = None  # the stream fills the queue: its steady state is the full step
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, threads = oracle_sample(w)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"1 chunk x 1 layer of the step ({t:.1f} s), scaled by "
                                          f"T x layers = {T * m.n_layers}; float64 numpy"}
        try:  # the same sample with the BLAS pool held to one thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                v1, t1, _ = oracle_sample(w)
            line["cpu_baseline"]["one_thread"] = {"value": v1, "unit": UNIT, "cores": 1,
                                                  "sample_s": round(t1, 2)}
        except ImportError:
            pass
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


def stream_summary(step_ms, occupancy, T, frames, wall_s, n_chunks):
    """Rates of one whole stream: steady state (steps with all T levels
    occupied: one chunk leaves per step) and whole stream (every chunk's frames
    over the host wall time from the first push to the last pop)."""
    steady = [t for t, n in zip(step_ms, occupancy) if n == T]
    out = {"chunks": n_chunks, "steps": len(step_ms), "wall_s": wall_s,
           "frames": n_chunks * frames, "whole_stream_frames_per_s": n_chunks * frames / wall_s,
           "steady_steps": len(steady)}
    if steady:
        med = statistics.median(steady)
        out["steady_ms_per_step"] = med
        out["steady_frames_per_s"] = frames / (med / 1e3)
    return out


def run_stream(args, w):
    """Whole streams of the workload's model, from the first push to the last
    pop (fill, steady state, drain), one per stream length, on one queue each:
    host pops every clean chunk to page-locked memory, device memory is sampled
    after every step.  The longest stream's steady state is the line's value."""
    import torch

    from chunked_fifo_denoising_b200 import Queue

    world, rank, local, dist = setup_rank()
    m, q = w.model, w.queue
    T, frames = q.T, q.frames_per_chunk
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cuda").manual_seed(1000 + rank)
    model, text = build_model(m, g, stream, args.neighbours)
    total = torch.cuda.mem_get_info()[1]
    lengths = sorted(set([int(x) for x in args.stream_lengths.split(",") if x] + [q.n_chunks]))
    runs = []
    clocks = Clocks(visible_index(local))
    for n in lengths:
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        queue = Queue(model, text, T, frames, q.lat_h, q.lat_w, n, ready_capacity=2, seed=3 + rank)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        peak_used = total - free1
        ho = torch.empty(queue.chunk_shape).pin_memory()
        step_ms, occupancy, popped = [], [], []
        if dist is not None:
            dist.barrier()
        t0 = time.perf_counter()
        while True:
            info = queue.inspect()
            if info["drained"]:
                break
            ts = time.perf_counter()
            queue.step(None)
            while True:
                st, cid = queue.try_pop(ho)
                if st != 0:
                    break
                popped.append(cid)
            queue.sync()
            step_ms.append((time.perf_counter() - ts) * 1e3)
            occupancy.append(info["n"])
            peak_used = max(peak_used, total - torch.cuda.mem_get_info()[0])
        wall = time.perf_counter() - t0
        assert popped == list(range(n)), "chunks must pop in push order"
        r = stream_summary(step_ms, occupancy, T, frames, wall, n)
        r.update({"queue_bytes": int(free0 - free1), "peak_device_bytes_used": int(peak_used)})
        runs.append(r)
        queue.close()
    ck = clocks.stop()
    head = runs[-1]
    peaks_equal = len({r["peak_device_bytes_used"] for r in runs}) == 1
    vals = max_over_ranks([head["wall_s"], head.get("steady_ms_per_step", 0.0)], dist, device="cuda")
    line = {"metric": METRIC, "mode": "stream",
            "value": world * frames / (vals[1] / 1e3) if vals[1] > 0 else None, "unit": UNIT,
            "n_gpus": world, "steps": head["steps"], "warmup": 0,
            "ms_per_step": vals[1], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic: seeded N(0,1) noise per chunk (device generator), "
                                     "N(0,1) prompt, N(0,0.02^2) random-init weights",
            "config": {"workload": w.name, "T": T, "chunks": q.n_chunks, "frames_per_chunk": frames,
                       "layers": m.n_layers, "dim": m.dim, "chunk_tokens": q.tokens_per_chunk(m),
                       "parallelism": f"replicas x{world}"},
            "whole_stream_frames_per_s": world * head["frames"] / vals[0],
            "streams": runs,
            "memory_flat_in_stream_length": peaks_equal,
            "memory_source": "cudaMemGetInfo (device-wide bytes in use) after dp_queue_init and after every step",
            "clocks": ck}
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--kernel-steps", type=int, default=2,
                    help="steps of the separate per-kernel timing pass")
    ap.add_argument("--stream", action="store_true",
                    help="run whole streams (fill, steady state, drain) instead of timing the "
                         "steady state alone; reports stream rates and peak device memory")
    ap.add_argument("--stream-lengths", default="32,64",
                    help="stream lengths (chunks) run besides the workload's own, with --stream")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan1.3b_480p")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--plateau", action="store_true",
                    help="also time the plateau of the workload's own stream length when it is "
                         "shorter than the queue (no push, no pop; rate = occupancy / T chunks per step)")
    ap.add_argument("--fill", default="steps", choices=["steps", "load"],
                    help="reach the steady state by T-1 real steps, or place it with "
                         "dp_queue_load_state (random latents and persisted K/V)")
    ap.add_argument("--qk-norm-rope", action="store_true",
                    help="per-head QK RMSNorm and 3-D rotary positions in self-attention")
    ap.add_argument("--neighbours", default="pred", choices=["pred", "both"],
                    help="self-attention neighbourhood: predecessor only, or also the successor")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    import synth
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.stream:
        return run_stream(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
