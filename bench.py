#!/usr/bin/env python
"""Benchmark of the VideoMLA latent-window attention hot path on B200.

One step = one rollout step of one attention layer at the Wan-1.3B geometry (hidden 1536,
12 heads, latent 192 + RoPE 32, 30 x 52 = 1560 tokens per latent frame, 21-frame window):
the 1560-token query frame attends to the window plus itself through the C ABI
(mla_window_attention: query projection with the frame's own latents, window attention, output
projection), then the frame joins the window (mla_cache_commit: its latents, which the query
projection already computed, move into their ring slot).  The same step with the frame's
latents recomputed by mla_cache_append is timed beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU under torchrun; every rank runs its own independent replicas
(no collective on the data path), the device time is the maximum over ranks and `value` is the
query tokens of all ranks divided by it (weak scaling).  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "latent-window attention query tokens/s and TFLOP/s (% of bf16 peak) per layer"
UNIT = "query tokens/s"
WORKLOAD = "wan_w21_q1"
FLOP_PER_QHK = 832          # 2*(192+32) for scores + 2*192 for P.c_kv, per (query, head, key)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024
REF_HEADS = 4              # heads per reference-arm step (of 12)


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--layers-cycle", type=int, default=12,
                   help="independent layer caches cycled so the step's inputs are not L2-resident")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=1560, help="query tokens in the oracle's timed sample")
    p.add_argument("--ncu-case", choices=("attention", "append", "steps", "dense"), default=None,
                   help="minimal launch sequence for an ncu capture (prints no benchmark line): "
                        "'attention' = fill + 2 steps, 'append' = 2 x 21-frame fill, 'steps' = warmup + K steps "
                        "(attention + commit), "
                        "'dense' = the dense per-head baseline over the 21-frame window (2 split-key calls, "
                        "then 1 one-pass call)")
    return p.parse_args(argv)


def run_ncu_case(args, local):
    """Short, fixed launch sequences for profiling under ncu (small device footprint)."""
    import torch

    import mla_synth
    from mla_latent_kv_window_b200 import build
    from mla_latent_kv_window_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    build.build()
    w = mla_synth.WORKLOADS[WORKLOAD]
    dims = dict(w.dims)
    F, W, hidden = w.F, w.window_frames, dims["hidden"]
    nq = w.query_frames * F
    if args.ncu_case == "dense":
        H, n_kv = dims["n_heads"], W * F + nq
        q = mla_synth.normal_bf16((1, nq, H, 128), 1.0, 1).to(dev)
        k = mla_synth.normal_bf16((1, n_kv, H, 128), 1.0, 2).to(dev)
        v = mla_synth.normal_bf16((1, n_kv, H, 128), 1.0, 3).to(dev)
        o = torch.empty_like(q)
        ws = torch.empty(B.mla_dense_workspace_bytes(1, nq, n_kv, H), dtype=torch.uint8, device=dev)
        for _ in range(2):
            B.mla_dense_attention(q, k, v, o, 0.0, None, workspace=ws)
        B.mla_dense_attention(q, k, v, o, 0.0, None)
        ok = B.mla_dense_sync() == 0
        print(json.dumps({"ncu_case": args.ncu_case, "device_status_ok": ok}))
        return 0 if ok else 1
    n_layers = 1 if args.ncu_case != "steps" else 2
    caches = []
    for layer in range(n_layers):
        wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, layer)).items()}
        caches.append(B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, W, w.query_frames))
    x_fill = mla_synth.make_hidden(1, W * F, hidden, mla_synth.fill_seed(w, 0)).to(dev)
    x = mla_synth.make_hidden(1, nq, hidden, mla_synth.chunk_seed(w, 0, 0)).to(dev)
    out = torch.empty_like(x)
    for c in caches:
        c.append(x_fill)
    if args.ncu_case == "append":
        caches[0].append(x_fill)
    else:
        n = 2 if args.ncu_case == "attention" else args.warmup + args.steps
        for s in range(n):
            c = caches[s % n_layers]
            c.attention(x, out)
            c.commit(w.query_frames)
    torch.cuda.synchronize()
    ok = all(B.mla_cache_sync(c.handle) == 0 for c in caches)
    print(json.dumps({"ncu_case": args.ncu_case, "device_status_ok": ok}))
    return 0 if ok else 1


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def sustained_peak():
    """Measured bf16 GEMM rate under the power cap (seconds-long loop), if recorded."""
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops_sustained"])
    except Exception:
        return None


# Device sources of each kernel whose ncu counters bench.py reports.
KERNEL_FILES = {"window_attn_kernel": ("ptx.cuh", "window_attn.cuh"),
                "append_fill": ("ptx.cuh", "gemm_tc.cuh")}


def kernel_source_hash(kernel: str) -> str:
    """Hash of what decides one profiled kernel: its device sources, and the launch constants of
    the host file (stage counts, tile shapes; the dense baseline's left out), with comments and
    blank lines removed, so that a comment, a host-only edit or a change to another kernel leaves
    the kernel, and the ncu counters taken on it, valid."""
    import re
    h = hashlib.sha256()
    for f in KERNEL_FILES[kernel] + ("mla_api.cu",):
        src = open(os.path.join(ROOT, "mla_latent_kv_window_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        lines = [l.rstrip() for l in src.splitlines() if l.strip()]
        if f.endswith(".cu"):
            lines = [l for l in lines if l.lstrip().startswith("constexpr") and "Dense" not in l]
        h.update("\n".join(lines).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        e = d[kernel]
        if e.get("source_hash") == kernel_source_hash(kernel):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, kept only for the timed window."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which: str):
        if which == "start":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self) -> dict:
        """End sampling; the record of the timed region marked with mark()."""
        time.sleep(0.15)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return self.window(self.t0, self.t1)

    def window(self, t0, t1) -> dict:
        """Median SM clock and the throttle reasons of the samples taken in [t0, t1] (host time)."""
        rows = []
        for t, line in list(self.lines):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((t, parts))
        inside = [r for t, r in rows if t0 is not None and t0 - 0.05 <= t <= (t1 or t) + 0.05]
        use = inside or [r for _, r in rows]
        sm = [float(r[1]) for r in use if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in use if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in use for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside)}


# ---------------------------------------------------------------------------- our arm
def run_ours(args, rank, local, world):
    import torch

    import mla_synth
    from mla_latent_kv_window_b200 import build, replicas
    from mla_latent_kv_window_b200 import binding as B

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    distributed = replicas.init("nccl")
    if rank == 0:
        build.build()
    replicas.barrier()
    B.load_library()

    w = mla_synth.WORKLOADS[WORKLOAD]
    dims = dict(w.dims)
    F, W = w.F, w.window_frames
    hidden = dims["hidden"]
    nq = w.query_frames * F
    n_keys = W * F + nq
    R = nq * dims["n_heads"]
    L = args.layers_cycle
    hbm_peak, tf_peak, peak_kind = peaks()
    tf_sust = sustained_peak()

    # Independent layer caches (distinct weights), each filled with a 21-frame window.
    caches = []
    for layer in range(L):
        wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, layer) + 1000 * rank).items()}
        c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, W, w.query_frames)
        x_fill = mla_synth.make_hidden(1, w.fill_frames * F, hidden, mla_synth.fill_seed(w, layer) + 1000 * rank).to(dev)
        c.append(x_fill)
        caches.append(c)
        del x_fill
    chunks = [mla_synth.make_hidden(1, nq, hidden, mla_synth.chunk_seed(w, 0, s) + 1000 * rank).to(dev) for s in range(4)]
    out = torch.empty(1, nq, hidden, dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    per_cache_bytes = B.mla_cache_device_bytes(caches[0].cfg)
    stream = torch.cuda.current_stream()

    def step(s):
        # One rollout step of one layer: the frame attends to the window plus itself, then its
        # latents (computed by the query projection) become part of the window.
        c = caches[s % L]
        x = chunks[s % 4]
        B.mla_window_attention(c.handle, x, w.query_frames, out, stream)
        B.mla_cache_commit(c.handle, w.query_frames, stream)

    def step_append(s):
        # The same step with the frame's latents recomputed from x by mla_cache_append.
        c = caches[s % L]
        x = chunks[s % 4]
        B.mla_window_attention(c.handle, x, w.query_frames, out, stream)
        B.mla_cache_append(c.handle, x, w.query_frames, stream)

    # ---- append roofline: the 21-frame fill, L2 flushed before each launch
    # Back-to-back fills alternating two 100 MB inputs (200 MB > the 126 MB L2, so every fill
    # reads its hidden states from HBM); CUDA events around 20 launches amortise launch latency.
    fill_cache = B.LatentWindowCache(dims, {k: v.to(dev) for k, v in mla_synth.make_weights(dims, 7).items()},
                                     w.frame_h, w.frame_w, W, w.query_frames)
    x_fills = [mla_synth.make_hidden(1, W * F, hidden, 99 + i).to(dev) for i in range(2)]
    for i in range(4):
        fill_cache.append(x_fills[i % 2])
    torch.cuda.synchronize()
    reps = 20
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(reps):
        B.mla_cache_append(fill_cache.handle, x_fills[i % 2], W, stream)
    f1.record(stream)
    torch.cuda.synchronize()
    append_ms = f0.elapsed_time(f1) / reps
    append_bytes = W * F * (hidden * 2 + 224 * 2) + 224 * hidden * 2
    fill_ok = B.mla_cache_sync(fill_cache.handle) == 0
    fill_cache.close()
    del x_fills

    # ---- main timed loop: events only around the K steps (no per-kernel events inside)
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    clocks.start()
    replicas.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark("start")
    e0.record(stream)
    for s in range(args.steps):
        step(args.warmup + s)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark("stop")
    replicas.barrier()
    ms_local = e0.elapsed_time(e1)
    ms = replicas.max_over_ranks(ms_local, dev)

    # ---- profiled pass: the same K steps again, CUDA events around every kernel launch on the
    # launching stream; gives the per-launch device time of each kernel (roofline).
    for c in caches:
        B.mla_cache_profile_enable(c.handle, True)
    replicas.barrier()
    torch.cuda.synchronize()
    for s in range(args.steps):
        step(args.warmup + args.steps + s)
    torch.cuda.synchronize()
    prof = {k: [0.0, 0] for k in B.KERNEL_NAMES}
    for c in caches:
        for k, (t, n) in B.mla_cache_profile_read(c.handle).items():
            prof[k][0] += t
            prof[k][1] += n
        B.mla_cache_profile_enable(c.handle, False)
    launches = 4 * args.steps   # each step launches Q-projection, attention, output projection, commit copy
    assert sum(n for _, n in prof.values()) == launches
    attn_ms = prof["attention"][0] / max(prof["attention"][1], 1)
    attn_ms = replicas.max_over_ranks(attn_ms, dev)

    # ---- the same K steps with the frame appended by recomputing its latents from x
    replicas.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        step_append(args.warmup + 2 * args.steps + s)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_append = replicas.max_over_ranks(e0.elapsed_time(e1), dev)

    tokens = world * nq * args.steps
    value = tokens / (ms / 1e3)
    attn_flop = FLOP_PER_QHK * R * n_keys
    attn_tflops = attn_flop / (attn_ms / 1e3) / 1e12
    step_tflops = attn_flop * args.steps / (ms_local / 1e3) / 1e12

    # ---- end to end through the public API with host buffers (pinned), copies inside the region.
    # A user's pipeline: each step's x is copied in on an H2D stream and its output copied out on
    # a D2H stream (PCIe is full duplex), double-buffered, so the copies of one step overlap the
    # kernels of its neighbours.  Every step still moves its own input and output.
    x_host = [ch.cpu().pin_memory() for ch in chunks]
    out_host = [torch.empty(1, nq, hidden, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty(1, nq, hidden, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    out_dev = [torch.empty(1, nq, hidden, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    compute = stream
    e2e_steps = max(1, min(args.steps, 400))
    ev = lambda: torch.cuda.Event()
    loaded = [ev(), ev()]
    computed = [ev(), ev()]
    drained = [ev(), ev()]
    used = [False, False]

    def e2e_step(s):
        i = s % 2
        c = caches[s % L]
        with torch.cuda.stream(h2d):
            if used[i]:
                h2d.wait_event(computed[i])          # step s-2 has finished reading x_dev[i]
            x_dev[i].copy_(x_host[s % 4], non_blocking=True)
            loaded[i].record(h2d)
        compute.wait_event(loaded[i])
        if used[i]:
            compute.wait_event(drained[i])           # step s-2's output has left out_dev[i]
        B.mla_window_attention(c.handle, x_dev[i], w.query_frames, out_dev[i], compute)
        B.mla_cache_commit(c.handle, w.query_frames, compute)
        computed[i].record(compute)
        with torch.cuda.stream(d2h):
            d2h.wait_event(computed[i])
            out_host[i].copy_(out_dev[i], non_blocking=True)
            drained[i].record(d2h)
        used[i] = True

    for s in range(min(args.warmup, 5)):
        e2e_step(s)
    torch.cuda.synchronize()
    replicas.barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(compute)
    h2d.wait_event(e2)
    for s in range(e2e_steps):
        e2e_step(s)
    compute.wait_event(drained[0])
    compute.wait_event(drained[1])
    e3.record(compute)
    torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks(e2.elapsed_time(e3), dev)
    e2e_value = world * nq * e2e_steps / (e2e_ms / 1e3)

    status_ok = all(B.mla_cache_sync(c.handle) == 0 for c in caches)
    for c in caches:
        c.close()
    caches.clear()
    torch.cuda.empty_cache()
    # Every rank takes part in the batched leg (its streams are sharded over the ranks).
    leg_t = {}
    t_a = time.time()
    batched = batched_leg(B, dev, stream, rank, world, tf_peak, hbm_peak)
    leg_t["wan_b4_w21_q3"] = (t_a, time.time())
    layout = layout_baseline(B, w, dims, dev, stream, attn_ms, attn_flop) if rank == 0 else None
    nxt = next_rows(B, dev) if rank == 0 else None
    t_a = time.time()
    rollout = rollout_leg(B, dev, stream, tf_peak) if rank == 0 else None
    leg_t["wan_30l_w21_q3_wrap"] = (t_a, time.time())
    tiny = tiny_leg(B, dev, stream) if rank == 0 else None
    clk = clocks.stop()
    for name, leg in (("wan_b4_w21_q3", batched.get("attention") if batched else None),
                      ("wan_30l_w21_q3_wrap", rollout)):
        if leg is not None:
            c = clocks.window(*leg_t[name])
            leg["clocks"] = {"sm_mhz": c["sm_mhz"], "reasons": c["reasons"], "samples": c["samples_in_timed_region"]}
            tf = leg.get("attention_tflops") or leg.get("attention_tflops_per_gpu")
            if tf and c["sm_mhz"]:
                # against what the tensor cores can do at the median sampled clock (8,192 flop/clk/SM)
                leg["attention_frac_of_tensor_rate_at_clock"] = round(
                    tf / (8192 * torch.cuda.get_device_properties(dev).multi_processor_count * c["sm_mhz"] * 1e-6), 4)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_rows)
        cpu["per_workload"] = cpu_workloads()
    replicas.barrier()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "precision": "bf16 hidden states, weights and output; fp16 cache planes, absorbed queries, P "
                         "and o_lat (tcgen05 kind::f16 operands); fp32 accumulation and softmax",
            "ms_per_step_append_recompute": round(ms_append / args.steps, 5),
            "data": "synthetic: seeded N(0,1) hidden states, N(0,1/fan_in) weights (no checkpoint)",
            "config": {
                "workload": f"{WORKLOAD}: Wan-1.3B-shaped layer, 21-frame latent window (32,760 cached tokens) "
                            f"+ one 1,560-token query frame",
                "hidden": hidden, "n_heads": dims["n_heads"], "d_latent": 192, "d_rope": 32, "d_nope": dims["d_nope"],
                "tokens_per_frame": F, "window_frames": W, "query_tokens": nq, "keys": n_keys, "batch": 1,
                "step": "mla_window_attention (Q-proj with the frame's latents + latent-window attention + "
                        "out-proj) then mla_cache_commit (the frame's latents moved into the ring slot)",
                "l2": f"inputs larger than L2: {L} independent layer caches cycled "
                      f"({L * per_cache_bytes / 2**20:.0f} MB > 126 MB)",
                "parallelism": f"replicas x{world} (no data-path collective)",
            },
            "attention_tflops": round(attn_tflops, 1),
            "pct_bf16_peak": round(100 * attn_tflops / tf_peak, 1),
            "step_attention_tflops": round(step_tflops, 1),
            "kernel_ms_per_launch": {k: round(t / max(n, 1), 5) for k, (t, n) in prof.items()},
            "kernel_timing": "per-launch CUDA events on the launching stream, in a second pass of the same K steps",
            "roofline": {
                "kernel": "window_attn_kernel", "bound": "tensor", "achieved": round(attn_tflops, 1),
                "peak": tf_peak, "unit": "TFLOP/s", "frac": round(attn_tflops / tf_peak, 4),
                "frac_of_sustained_peak": (round(attn_tflops / tf_sust, 4) if tf_sust else None),
                "traffic": measured_traffic("window_attn_kernel"),
                "peak_source": f"{peak_kind} bf16 (burst)",
                "algorithmic": f"{FLOP_PER_QHK} flop per (query, head, key) x {R} rows x {n_keys} keys "
                               f"= {attn_flop / 1e9:.1f} GFLOP per launch",
            },
            "projection_rooflines": projection_rooflines(prof, dims, nq, tf_peak, peak_kind),
            "append_roofline": {
                "kernel": "tc_gemm_kernel<224,latent> (21-frame fill; 20 back-to-back launches alternating two 100 MB inputs)",
                "bound": "hbm", "status_ok": fill_ok,
                "achieved": round(append_bytes / (append_ms / 1e3) / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(append_bytes / (append_ms / 1e3) / 1e9 / hbm_peak, 4),
                "ms_per_launch": round(append_ms, 5), "traffic": measured_traffic("append_fill"),
                "algorithmic": f"{W * F} tokens x (3072 B in + 448 B out) + 688,128 B weights = {append_bytes / 1e6:.1f} MB",
                "peak_source": f"{peak_kind} HBM copy",
            },
            "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": nq * hidden * 2,
                    "d2h_bytes_per_step": nq * hidden * 2, "steps": e2e_steps,
                    "pipeline": "pinned host buffers; H2D and D2H streams double-buffered against the compute stream"},
            "gpu_launches": int(launches),
            "device_status_ok": status_ok,
            "clocks": clk,
        }
        line["workloads"] = {k: v for k, v in (("tiny", tiny), ("wan_30l_w21_q3_wrap", rollout),
                                               ("wan_b4_w21_q3", batched.get("attention") if batched else None))
                             if v is not None}
        if batched:
            line["append_roofline_b4"] = batched["fill"]
        if layout is not None:
            line["layout_baseline"] = layout
        if nxt is not None:
            line["next_rows"] = nxt
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    replicas.shutdown()


def projection_rooflines(prof, dims, nq, tf_peak, peak_kind):
    """The two projections of a step against the tensor peak, from the profiled pass's per-launch
    CUDA-event times (each including its kernel boundary).  Algorithmic FLOPs are the absorbed
    form's: the query launch 2 n_q hidden (n_h (d_latent + d_rope) + d_latent + d_rope) (the
    queries and the chunk latents), the output launch 2 n_q hidden n_h d_latent; the query
    launch's executed FLOPs (W_Q, W_QR, W_DKV, W_KR, then the W_UK product on an fp16 pair) are
    given beside them."""
    hid, nh, dc, dr, dn = dims["hidden"], dims["n_heads"], dims["d_latent"], dims["d_rope"], dims["d_nope"]
    q_alg = 2.0 * nq * hid * (nh * (dc + dr) + dc + dr)
    q_exec = 2.0 * nq * hid * (nh * (dn + dr) + dc + dr) + 2.0 * nq * nh * (2 * dn) * dc
    o_alg = 2.0 * nq * hid * nh * dc
    out = {}
    for name, kern, flop, extra in (("query", "qproj", q_alg, {"executed_gflop": round(q_exec / 1e9, 2)}),
                                    ("output", "oproj", o_alg, {})):
        t, n = prof.get(kern, (0.0, 0))
        if not n:
            continue
        ms = t / n
        tf = flop / (ms / 1e3) / 1e12
        out[name] = dict({"ms_per_launch": round(ms, 5), "gflop": round(flop / 1e9, 2),
                          "achieved": round(tf, 1), "peak": tf_peak, "unit": "TFLOP/s",
                          "frac": round(tf / tf_peak, 4), "bound": "tensor"}, **extra)
    out["peak_source"] = f"{peak_kind} bf16 (burst)"
    return out


def _profiled_attention_ms(B, caches, fn, warm=1, reps=3):
    """Run fn (warm + reps times) with per-launch events on every cache; returns the per-launch
    device ms of each kernel kind over the timed reps, and the launch counts."""
    import torch
    for c in caches:
        B.mla_cache_profile_enable(c.handle, True)
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    for c in caches:
        B.mla_cache_profile_read(c.handle)
    for _ in range(reps):
        fn()
    torch.cuda.synchronize()
    tot = {k: [0.0, 0] for k in B.KERNEL_NAMES}
    for c in caches:
        for k, (t, n) in B.mla_cache_profile_read(c.handle).items():
            tot[k][0] += t
            tot[k][1] += n
        B.mla_cache_profile_enable(c.handle, False)
    return {k: (t / n if n else 0.0, n) for k, (t, n) in tot.items()}


def rollout_leg(B, dev, stream, tf_peak, reps=2):
    """The 30-layer rollout of the Wan-1.3B geometry: 30 layers with independent weights, each
    with a 21-frame ring that has wrapped (24 frames appended, the oldest 3 evicted); one 3-frame
    chunk (4,680 query tokens) is denoised in 4 steps (every step runs all 30 layers against
    the same caches), then its latents are committed to every layer's window.  Reported per
    layer-step: query tokens/s over the whole chunk (120 layer-steps + 30 commits), and the
    attention kernel's TFLOP/s over 37,440 keys."""
    import torch

    import mla_synth
    w = mla_synth.WORKLOADS["wan_30l_w21_q3_wrap"]
    dims = dict(w.dims)
    F, hidden, Q = w.F, dims["hidden"], w.query_frames
    caches = []
    for layer in range(w.layers):
        wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, layer)).items()}
        c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, w.window_frames, Q)
        c.append(mla_synth.make_hidden(1, w.fill_frames * F, hidden, mla_synth.fill_seed(w, layer)).to(dev))
        caches.append(c)
    xs = [mla_synth.make_hidden(1, Q * F, hidden, mla_synth.chunk_seed(w, 0, st)).to(dev) for st in range(w.steps)]
    out = torch.empty_like(xs[0])

    def chunk():
        for st in range(w.steps):
            for c in caches:
                B.mla_window_attention(c.handle, xs[st], Q, out, stream)
        for c in caches:
            B.mla_cache_commit(c.handle, Q, stream)

    chunk()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        chunk()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    prof = _profiled_attention_ms(B, caches, chunk, warm=0, reps=1)
    ok = all(B.mla_cache_sync(c.handle) == 0 for c in caches)
    _, valid = caches[0].state()
    for c in caches:
        c.close()
    nq = Q * F
    keys = valid * F + nq
    layer_steps = w.layers * w.steps
    a_ms = prof["attention"][0]
    flop = FLOP_PER_QHK * nq * dims["n_heads"] * keys
    return {"workload": "30 Wan-1.3B-shaped layers, 21-frame wrapped ring, 3-frame chunk (4,680 query tokens) "
                        "x 4 denoising steps, then the chunk committed to every layer",
            "keys": keys, "query_tokens_per_layer_step": nq, "layer_steps_per_chunk": layer_steps,
            "ms_per_chunk": round(ms, 3),
            "query_tokens_per_s_per_layer_step": round(nq * layer_steps / (ms / 1e3), 1),
            "attention_ms": round(a_ms, 4), "attention_tflops": round(flop / (a_ms / 1e3) / 1e12, 1),
            "attention_frac_of_peak": round(flop / (a_ms / 1e3) / 1e12 / tf_peak, 4),
            "kernel_ms_per_launch": {k: round(t, 5) for k, (t, n) in prof.items() if n},
            "status_ok": ok}


def batched_leg(B, dev, stream, rank, world, tf_peak, hbm_peak, reps=5):
    """B = 4 independent streams (per-stream hidden-state scale in [0.5, 2]), each a 21-frame
    window and a 3-frame chunk, sharded over the ranks (replicas.shard): each rank holds a cache
    of its own streams, no collective on the data path.  Also the fill of those windows
    (mla_cache_append of 21 frames per stream), the append's HBM roofline point at B = 4."""
    import torch

    import mla_synth
    from mla_latent_kv_window_b200 import replicas
    w = mla_synth.WORKLOADS["wan_b4_w21_q3"]
    dims = dict(w.dims)
    F, hidden, Q, W = w.F, dims["hidden"], w.query_frames, w.window_frames
    mine = list(replicas.shard(w.batch, rank, world))
    nb = len(mine)
    fill_ms = attn_call_ms = a_ms = 0.0
    ok = True
    if nb:
        scales = mla_synth.stream_scales(w.batch, w.seed)
        wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0)).items()}
        c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, W, Q, batch=nb)
        x_fill = mla_synth.make_hidden(w.batch, W * F, hidden, mla_synth.fill_seed(w, 0), scales)[mine].to(dev)
        c.append(x_fill)
        torch.cuda.synchronize()
        # Fill roofline: x is 4 x 32,760 x 1536 bf16 = 403 MB, larger than L2, so every fill
        # reads it from HBM.
        fill_ms = _event_ms(lambda: B.mla_cache_append(c.handle, x_fill, W, stream), stream, reps=reps, warm=2)
        del x_fill
        x = mla_synth.make_hidden(w.batch, Q * F, hidden, mla_synth.chunk_seed(w, 0, 0), scales)[mine].to(dev)
        out = torch.empty_like(x)
        attn_call_ms = _event_ms(lambda: B.mla_window_attention(c.handle, x, Q, out, stream), stream, reps=reps, warm=2)
        prof = _profiled_attention_ms(B, [c], lambda: B.mla_window_attention(c.handle, x, Q, out, stream))
        a_ms = prof["attention"][0]
        ok = B.mla_cache_sync(c.handle) == 0
        c.close()
    fill_ms = replicas.max_over_ranks(fill_ms, dev)
    attn_call_ms = replicas.max_over_ranks(attn_call_ms, dev)
    a_ms = replicas.max_over_ranks(a_ms, dev)
    nq, keys = Q * F, W * F + Q * F
    per_rank_streams = max(len(replicas.shard(w.batch, r, world)) for r in range(world))
    flop = FLOP_PER_QHK * per_rank_streams * nq * dims["n_heads"] * keys
    fill_bytes = per_rank_streams * W * F * (hidden * 2 + 224 * 2) + 224 * hidden * 2
    return {
        "attention": {
            "workload": f"B = 4 streams sharded over {world} GPU(s) ({per_rank_streams} per GPU at most), "
                        f"21-frame window, 3-frame chunk, per-stream scale in [0.5, 2]",
            "keys": keys, "query_tokens": w.batch * nq, "call_ms": round(attn_call_ms, 4),
            "query_tokens_per_s": round(w.batch * nq / (attn_call_ms / 1e3), 1),
            "attention_ms": round(a_ms, 4),
            "attention_tflops_per_gpu": round(flop / (a_ms / 1e3) / 1e12, 1) if a_ms else None,
            "attention_frac_of_peak": round(flop / (a_ms / 1e3) / 1e12 / tf_peak, 4) if a_ms else None,
            "status_ok": ok},
        "fill": {
            "kernel": "tc_gemm_kernel<224,latent> (21-frame fill of the B = 4 streams, x from HBM)",
            "bound": "hbm", "ms_per_launch": round(fill_ms, 5),
            "achieved": round(fill_bytes / (fill_ms / 1e3) / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(fill_bytes / (fill_ms / 1e3) / 1e9 / hbm_peak, 4),
            "algorithmic": f"{per_rank_streams} x 32,760 tokens x (3072 B in + 448 B out) + 688,128 B weights "
                           f"= {fill_bytes / 1e6:.1f} MB per GPU",
            "status_ok": ok},
    }


def graph_replay_ms(B, c, x, out, reps=20):
    """Per-call ms of one attention call on cache c, launched directly and as a CUDA-graph replay
    (the call captured once with static x and out buffers; valid while the cache state it saw at
    capture is unchanged, i.e. for the denoising steps of one chunk)."""
    import torch
    st = torch.cuda.current_stream()
    direct = _event_ms(lambda: c.attention(x, out, st), st, reps=reps)
    side = torch.cuda.Stream()
    side.wait_stream(st)
    with torch.cuda.stream(side):
        c.attention(x, out)
    st.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        c.attention(x, out)
    replay = _event_ms(g.replay, st, reps=reps)
    del g
    return direct, replay


def tiny_leg(B, dev, stream):
    """The small workload (4 x 6 frames, 2-frame window, one query frame): launch-bound."""
    import torch

    import mla_synth
    w = mla_synth.WORKLOADS["tiny"]
    dims = dict(w.dims)
    wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0)).items()}
    c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, w.window_frames, w.query_frames)
    c.append(mla_synth.make_hidden(1, w.fill_frames * w.F, dims["hidden"], mla_synth.fill_seed(w, 0)).to(dev))
    x = mla_synth.make_hidden(1, w.F, dims["hidden"], mla_synth.chunk_seed(w, 0, 0)).to(dev)
    out = torch.empty_like(x)
    ms = _event_ms(lambda: B.mla_window_attention(c.handle, x, 1, out, stream), stream, reps=20)
    direct, replay = graph_replay_ms(B, c, x, out)
    ok = B.mla_cache_sync(c.handle) == 0
    c.close()
    return {"workload": "4 x 6-token frames, 2-frame window, one query frame (72 keys)", "call_ms": round(ms, 4),
            "query_tokens_per_s": round(w.F / (ms / 1e3), 1), "status_ok": ok,
            "cuda_graph": {"direct_call_ms": round(direct, 4), "graph_replay_ms": round(replay, 4)},
            "note": "launch-bound: three kernels for 24 query tokens"}


def _event_ms(fn, stream, reps=10, warm=3):
    import torch
    for _ in range(warm):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def layout_baseline(B, w, dims, dev, stream, latent_ms, latent_flop):
    """The layout comparison of the long-window workload: dense per-head 12 x 128 K/V attention at
    the 21-frame window (same keys as the latent kernel above), and the latent kernel at a
    63-frame window (98,280 cached tokens, about as many bytes as 4.6 dense frames)."""
    import torch

    import mla_synth
    F, nq = w.F, w.query_frames * w.F
    n_kv = w.window_frames * F + nq
    H = dims["n_heads"]
    q = mla_synth.normal_bf16((1, nq, H, 128), 1.0, 1).to(dev)
    k = mla_synth.normal_bf16((1, n_kv, H, 128), 1.0, 2).to(dev)
    v = mla_synth.normal_bf16((1, n_kv, H, 128), 1.0, 3).to(dev)
    o = torch.empty_like(q)
    ws = torch.empty(B.mla_dense_workspace_bytes(1, nq, n_kv, H), dtype=torch.uint8, device=dev)
    dense_ms = _event_ms(lambda: B.mla_dense_attention(q, k, v, o, 0.0, stream, workspace=ws), stream)
    dense_1pass_ms = _event_ms(lambda: B.mla_dense_attention(q, k, v, o, 0.0, stream), stream)
    dense_ok = B.mla_dense_sync(stream) == 0
    dense_flop = 4 * nq * n_kv * 128 * H
    del q, k, v, o, ws
    w63 = mla_synth.WORKLOADS["wan_w63_q1"]
    wts = {kk: vv.to(dev) for kk, vv in mla_synth.make_weights(dims, mla_synth.weight_seed(w63, 0)).items()}
    c63 = B.LatentWindowCache(dims, wts, w63.frame_h, w63.frame_w, w63.window_frames, 1)
    c63.append(mla_synth.make_hidden(1, 63 * F, dims["hidden"], mla_synth.fill_seed(w63, 0)).to(dev))
    x = mla_synth.make_hidden(1, F, dims["hidden"], mla_synth.chunk_seed(w63, 0, 0)).to(dev)
    out = torch.empty_like(x)
    B.mla_cache_profile_enable(c63.handle, True)
    for _ in range(3):
        c63.attention(x, out)
    torch.cuda.synchronize()
    B.mla_cache_profile_read(c63.handle)
    for _ in range(10):
        c63.attention(x, out)
    torch.cuda.synchronize()
    p63 = B.mla_cache_profile_read(c63.handle)
    ok63 = B.mla_cache_sync(c63.handle) == 0
    c63.close()
    a63_ms = p63["attention"][0] / max(p63["attention"][1], 1)
    keys63 = 63 * F + F
    flop63 = FLOP_PER_QHK * nq * H * keys63
    cache_bytes = lambda per_tok, frames: frames * F * per_tok * 2
    return {
        "dense_per_head_21_frames": {
            "kernel": "dense_attn_kernel (12 x 128 K and V per token, bf16), split keys + combine",
            "keys": n_kv,
            "ms": round(dense_ms, 4), "tflops": round(dense_flop / (dense_ms / 1e3) / 1e12, 1),
            "one_pass_ms": round(dense_1pass_ms, 4),
            "query_tokens_per_s": round(nq / (dense_ms / 1e3), 1),
            "cache_bytes_per_layer": cache_bytes(3072, w.window_frames), "status_ok": dense_ok},
        "latent_21_frames": {
            "ms": round(latent_ms, 4), "tflops": round(latent_flop / (latent_ms / 1e3) / 1e12, 1),
            "query_tokens_per_s": round(nq / (latent_ms / 1e3), 1),
            "cache_bytes_per_layer": cache_bytes(224, w.window_frames)},
        "latent_63_frames": {
            "keys": keys63, "ms": round(a63_ms, 4), "tflops": round(flop63 / (a63_ms / 1e3) / 1e12, 1),
            "query_tokens_per_s": round(nq / (a63_ms / 1e3), 1),
            "cache_bytes_per_layer": cache_bytes(224, 63), "status_ok": ok63},
        "note": "dense counts 512 flop per (query, head, key); latent 832 (absorbed scores + P.c_kv)",
    }


def next_rows(B, dev):
    """Per-launch times of the rows after the main path: the paper-default dims (96/32 split,
    d_q = 768, RoPE (6,5,5) pairs) on the 21-frame one-frame step, and 1 sink frame + a 6-frame
    window with 3-frame chunks (the long-rollout configuration)."""
    import torch

    import mla_synth
    res = {}
    for name, chunk_frames in (("paper_w21_q1", 1), ("sink_w6_q3", 3)):
        w = mla_synth.WORKLOADS[name]
        dims = dict(w.dims)
        F = w.F
        wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0)).items()}
        c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, w.window_frames, chunk_frames,
                                sink_frames=w.sink_frames)
        c.append(mla_synth.make_hidden(1, w.fill_frames * F, dims["hidden"], mla_synth.fill_seed(w, 0)).to(dev))
        x = mla_synth.make_hidden(1, chunk_frames * F, dims["hidden"], mla_synth.chunk_seed(w, 0, 0)).to(dev)
        out = torch.empty_like(x)
        B.mla_cache_profile_enable(c.handle, True)
        for _ in range(3):
            c.attention(x, out)
        torch.cuda.synchronize()
        B.mla_cache_profile_read(c.handle)
        reps = 10
        for _ in range(reps):
            c.attention(x, out)
        torch.cuda.synchronize()
        prof = B.mla_cache_profile_read(c.handle)
        ok = B.mla_cache_sync(c.handle) == 0
        _, valid = c.state()
        c.close()
        nq = chunk_frames * F
        keys = valid * F + nq
        a_ms = prof["attention"][0] / max(prof["attention"][1], 1)
        call_ms = sum(t for t, _ in prof.values()) / reps
        flop = FLOP_PER_QHK * nq * dims["n_heads"] * keys
        res[name] = {
            "keys": keys, "query_tokens": nq,
            "attention_ms": round(a_ms, 4), "attention_tflops": round(flop / (a_ms / 1e3) / 1e12, 1),
            "call_ms": round(call_ms, 4), "query_tokens_per_s": round(nq / (call_ms / 1e3), 1),
            "kernel_ms_per_launch": {k: round(t / max(n, 1), 5) for k, (t, n) in prof.items() if n},
            "status_ok": ok,
        }
    res["note"] = ("attention TFLOP/s at 832 flop per (query, head, key) over the valid keys (sink "
                   "padding rows excluded); call = query projection + attention + output projection")
    res["reconstruct_vs_absorbed"] = reconstruct_crossover(B, dev)
    return res


def reconstruct_crossover(B, dev):
    """Absorbed kernel vs reconstruct-then-dense on the paper-default dims over the 21-frame
    window, for 1-, 2- and 3-frame chunks (whole calls, CUDA events).  The dense form pays a
    per-call reconstruction of every key and then 512 flop per (query, head, key) instead of 832;
    a straight-line fit of both call times in the query count gives where they cross."""
    import numpy as np
    import torch

    import mla_synth
    w = mla_synth.WORKLOADS["paper_w21_q1"]
    dims = dict(w.dims)
    F = w.F
    wts = {k: v.to(dev) for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0)).items()}
    c = B.LatentWindowCache(dims, wts, w.frame_h, w.frame_w, w.window_frames, 3)
    c.append(mla_synth.make_hidden(1, w.fill_frames * F, dims["hidden"], mla_synth.fill_seed(w, 0)).to(dev))
    stream = torch.cuda.current_stream()
    rows = []
    for nf in (1, 2, 3):
        x = mla_synth.make_hidden(1, nf * F, dims["hidden"], mla_synth.chunk_seed(w, 0, nf)).to(dev)
        out = torch.empty_like(x)
        t_abs = _event_ms(lambda: c.attention(x, out), stream)
        t_rec = _event_ms(lambda: c.attention_reconstruct(x, out), stream)
        rows.append({"query_tokens": nf * F, "keys": w.window_frames * F + nf * F,
                     "absorbed_ms": round(t_abs, 4), "reconstruct_dense_ms": round(t_rec, 4)})
    ok = B.mla_cache_sync(c.handle) == 0
    c.close()
    n = np.array([r["query_tokens"] for r in rows], dtype=np.float64)
    ta = np.array([r["absorbed_ms"] for r in rows])
    tr = np.array([r["reconstruct_dense_ms"] for r in rows])
    (ba, aa), (br, ar) = np.polyfit(n, ta, 1), np.polyfit(n, tr, 1)
    cross = (ar - aa) / (ba - br) if ba != br else None
    return {"workload": "paper dims (96 + 32 per head, d_q = 768, RoPE (6,5,5)), 21-frame window",
            "calls": rows, "status_ok": ok,
            "fit_ms": {"absorbed": [round(aa, 4), round(ba * 1e3, 5)],
                       "reconstruct_dense": [round(ar, 4), round(br * 1e3, 5)],
                       "form": "[intercept ms, ms per 1000 query tokens]"},
            "crossover_query_tokens": (round(float(cross), 1) if cross is not None else None),
            "note": "reconstruct-then-dense is faster above the crossover when the crossover is "
                    "positive and its slope is smaller; the window's keys are reconstructed "
                    "every call"}


# ---------------------------------------------------------------------------- the oracle on CPU
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_layer(w, rank=0):
    import mla_synth
    from oracle import OracleLayer
    dims = dict(w.dims)
    dims.update(frame_h=w.frame_h, frame_w=w.frame_w, window_frames=w.window_frames)
    orc = OracleLayer(dims, mla_synth.make_weights(dict(w.dims), mla_synth.weight_seed(w, 0) + 1000 * rank))
    orc.append(mla_synth.make_hidden(1, w.fill_frames * w.F, dims["hidden"], mla_synth.fill_seed(w, 0) + 1000 * rank)[0])
    return orc


def cpu_baseline(w, rows: int) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of one step: `rows` query tokens, all
    heads, all 34,320 keys (window filled beforehand, not timed)."""
    import numpy as np

    import mla_synth
    orc = _oracle_layer(w)
    x = mla_synth.make_hidden(1, w.query_frames * w.F, w.dim("hidden"), mla_synth.chunk_seed(w, 0, 0))[0]
    sel = np.linspace(0, x.shape[0] - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    orc.attention(x, rows=sel)
    dt = time.perf_counter() - t0
    return {"value": round(rows / dt, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{rows} of {x.shape[0]} query tokens of one step (12 heads, {w.window_frames * w.F + x.shape[0]} keys, "
                      f"float64 NumPy, per-head K/V materialised)"}


def cpu_workloads(rows: int = 96) -> dict:
    """The oracle on a bounded sample of each other workload: `rows` query tokens (all heads,
    all keys) of one attention call, window filled beforehand (not timed)."""
    import numpy as np

    import mla_synth
    from oracle import OracleLayer
    res = {}
    for name in ("tiny", "wan_30l_w21_q3_wrap", "wan_b4_w21_q3", "wan_w63_q1"):
        w = mla_synth.WORKLOADS[name]
        dims = dict(w.dims)
        dims.update(frame_h=w.frame_h, frame_w=w.frame_w, window_frames=w.window_frames)
        orc = OracleLayer(dims, mla_synth.make_weights(dict(w.dims), mla_synth.weight_seed(w, 0)))
        scales = mla_synth.stream_scales(w.batch, w.seed) if w.stream_scale else None
        orc.append(mla_synth.make_hidden(w.batch, w.fill_frames * w.F, dims["hidden"],
                                         mla_synth.fill_seed(w, 0), scales)[0])
        x = mla_synth.make_hidden(w.batch, w.query_frames * w.F, dims["hidden"],
                                  mla_synth.chunk_seed(w, 0, 0), scales)[0]
        n = min(rows, x.shape[0])
        sel = np.linspace(0, x.shape[0] - 1, n).astype(np.int64)
        t0 = time.perf_counter()
        orc.attention(x, rows=sel)
        dt = time.perf_counter() - t0
        keys = len(orc.active_frames()) * w.F + x.shape[0]
        res[name] = {"value": round(n / dt, 3), "unit": UNIT, "seconds": round(dt, 2),
                     "sample": f"{n} of {x.shape[0]} query tokens of one call (stream 0, all heads, {keys} keys)"}
    return res


def run_reference(args, rank, world):
    """The oracle timed on the host cores as the reference arm (rank 0 only).

    One step is the benchmarked step's work in the oracle: append the previous query frame (the
    window slides by one frame), then attend all 1,560 query tokens of the next frame over the
    whole window and the frame itself, for REF_HEADS of the 12 heads (a different group each
    step).  Heads are independent and cost the same (each materialises its own K and V over all
    keys), so a step is a third of a full step's work in the same proportions, and the value, in
    query-token equivalents (tokens x heads / 12) per second, measures the same rate as the
    cpu_baseline leg's full step."""
    if rank != 0:
        return
    import mla_synth
    w = mla_synth.WORKLOADS[WORKLOAD]
    orc = _oracle_layer(w)
    nq = w.query_frames * w.F
    n_heads = w.dim("n_heads")
    chunks = [mla_synth.make_hidden(1, nq, w.dim("hidden"), mla_synth.chunk_seed(w, 0, s))[0] for s in range(4)]

    def step(s):
        heads = [(s * REF_HEADS + i) % n_heads for i in range(REF_HEADS)]
        orc.attention(chunks[s % 4], heads=heads)
        orc.append(chunks[s % 4])

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(args.warmup + s)
    dt = time.perf_counter() - t0
    tok = args.steps * nq * REF_HEADS / n_heads
    value = tok / dt
    cores = blas_threads()
    sample = (f"per step: 1-frame append + all {nq} query tokens x {REF_HEADS} of {n_heads} heads over all "
              f"{w.window_frames * w.F + nq} keys (float64 NumPy oracle, per-head K/V materialised); "
              f"value counts tokens*heads/{n_heads} token-equivalents")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / max(args.steps, 1), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: Wan-1.3B-shaped layer, 21-frame latent window + one 1,560-token query frame"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    args = parse_args(argv)
    from mla_latent_kv_window_b200.replicas import env_rank
    rank, local, world = env_rank()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.ncu_case:
        return run_ncu_case(args, local)
    return run_ours(args, rank, local, world)


if __name__ == "__main__":
    sys.exit(main() or 0)
