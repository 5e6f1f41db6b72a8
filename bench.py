#!/usr/bin/env python
"""Benchmark: Z-Image S3-DiT full transformer forward at 4,128 tokens on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full forward (2 noise-refiner + 2 context-refiner + 30 main
blocks, embedders and final layer) of a 1024x1024 image (latent 16x128x128 ->
4,096 image tokens) with 32 text tokens, batch 1, on random-init bf16 weights
(6,154,908,736 parameters, seeded) resident in HBM.  The value is algorithmic
TFLOP/s (per block 8SD^2 + 6SDF + 4S^2D, plus embedders and final layer).

--gpus N > 1 runs N independent replicas (one process per GPU, launched by
torch.distributed.run); the forward has no exchange step, so there is no
data-path collective: barriers and the max-over-ranks timing use NCCL.

After the headline timing the same run also times, on the same resident weights,
the forward with e4m3 projections (e4m3_forwards), the 8-step Turbo loop at
4,096 + 128 tokens replayed as one CUDA graph, and one CFG step at 2048x2048
(batch 2 x 16,896 tokens) (workloads); --no-e4m3 / --no-workloads skip them.

--impl reference times the CPU oracle (NumPy, fp64) on the host cores, each
step one main block of the same 4,128-token workload (a bounded sample).

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import zimage_inputs as zi  # noqa: E402

METRIC = "DiT forward ms & TFLOP/s at 4,128 tokens; % of B200 bf16 tensor peak"
WORKLOAD = ("full stack one forward: 2 context-refiner + 2 noise-refiner + 30 main blocks, "
            "1024x1024 -> 4,096 image + 32 text = 4,128 tokens, batch 1")
LAT_H = LAT_W = 128
S_TXT = 32
T_VALUE = 0.5
SEED = 0
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The pages' own number for this workload (Z-Image-Turbo repackaged for H3ddle, "Measured
# performance"): one complete 4,128-token transformer forward in 22.5 s (input-major int8
# weights, Apple M1 Pro), i.e. FORWARD_FLOPS / 22.5 s.  Another machine and precision:
# context for vs_baseline, not the target.
PAGES_FORWARD_S = 22.5


def block_flops(S: int, D: int, F: int) -> float:
    return 8.0 * S * D * D + 6.0 * S * D * F + 4.0 * S * S * D


def forward_flops(d: zi.Dims, s_img: int, s_txt: int, batch: int = 1) -> float:
    D, F = d.dim, d.ffn
    S = s_img + s_txt
    f = d.n_noise * block_flops(s_img, D, F) + d.n_ctx * block_flops(s_txt, D, F) + d.n_main * block_flops(S, D, F)
    f += 2.0 * s_img * d.patch_dim * D + 2.0 * s_txt * d.cap_dim * D + 2.0 * s_img * D * d.patch_dim
    return batch * f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash(files) -> str:
    """Hash of the CUDA sources a kernel is built from (names under the package's csrc/),
    over the code only: comments and whitespace are dropped, so editing a comment does
    not mark recorded counters as stale, while any change to the code does."""
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "stream_diffusion_transformer_b200", "csrc")
    for name in sorted(files):
        with open(os.path.join(cdir, name)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)   # block comments
        text = re.sub(r"//[^\n]*", " ", text)                  # line comments
        h.update(name.encode() + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json), or None
    if there is none or the kernel's sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        rec = json.load(fh)
    e = rec.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as fh:
            for line in fh:
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        mx = float(rows[0][2])
        load = [float(r[1]) for r in rows if float(r[3]) > 250.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample():
    """The CPU oracle's bounded sample: one main block of the 4,128-token workload (fp64)."""
    from oracle import zimage_ref as ref
    d = zi.FULL
    s_img = (LAT_H // 2) * (LAT_W // 2)
    S = s_img + S_TXT
    bits = zi.make_weights(d, seed=SEED, keys=[k for k, _, _ in zi.block_specs("layers.0", d, True)], threads=8)
    W = ref.Weights(bits)
    x = zi.make_stream(d, 1, S, seed=SEED)[0].astype(np.float64)
    c = zi.make_cond(d, 1, seed=SEED)[0].astype(np.float64)
    ang = ref.rope_angles(ref.position_ids(S_TXT, LAT_H // 2, LAT_W // 2), d.rope_axes)

    def step():
        return ref.block_forward(x, W, "layers.0", d, ang, c)

    return step, block_flops(S, d.dim, d.ffn), f"one main block (full width, {S} tokens, fp64 NumPy)"


def run_oracle_workload(args):
    """Times the CPU oracle (fp64 NumPy) on the small configurations, on this host's
    cores: the tiny model's whole forward, one full-width main block at 1,152 tokens
    (all BLAS threads and one), and one main block at 4,128 tokens, from which a full
    4,128-token forward is extrapolated.  Prints one JSON line."""
    from threadpoolctl import threadpool_limits

    from oracle import zimage_ref as ref

    def timed(fn, min_s=2.0):
        fn()
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            dt = time.perf_counter() - t0
            if dt >= min_s:
                return dt / n

    out = {"workload": "CPU oracle timings (fp64 NumPy)", "host_cpus": os.cpu_count(),
           "affinity_cpus": len(os.sched_getaffinity(0)), "blas_threads": blas_threads()}
    # the tiny model, whole forward (64 image + 32 text tokens)
    d = zi.TINY
    W = ref.Weights(zi.make_weights(d, seed=SEED))
    lat = zi.make_latent(d, 1, 16, 16, seed=SEED).astype(np.float64)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 32, seed=SEED)).astype(np.float64)
    tt = np.array([T_VALUE])
    sec = timed(lambda: ref.model_forward(lat, tt, txt, W, d))
    fl = forward_flops(d, 64, 32)
    out["tiny_model_forward"] = {"ms": sec * 1e3, "gflops": fl / sec / 1e9, "flops": fl}
    # one full-width main block at 1,024 + 128 and at 4,096 + 32 tokens
    d = zi.FULL
    W = ref.Weights(zi.make_weights(d, seed=SEED, keys=[k for k, _, _ in zi.block_specs("layers.0", d, True)],
                                    threads=8))
    for name, (gh, gw, st) in {"block_1152": (32, 32, 128), "block_4128": (64, 64, S_TXT)}.items():
        S = gh * gw + st
        x = zi.make_stream(d, 1, S, seed=SEED)[0].astype(np.float64)
        c = zi.make_cond(d, 1, seed=SEED)[0].astype(np.float64)
        ang = ref.rope_angles(ref.position_ids(st, gh, gw), d.rope_axes)
        fl = block_flops(S, d.dim, d.ffn)
        sec = timed(lambda: ref.block_forward(x, W, "layers.0", d, ang, c))
        out[name] = {"tokens": S, "ms": sec * 1e3, "gflops": fl / sec / 1e9, "threads": blas_threads()}
        if name == "block_1152":
            with threadpool_limits(limits=1, user_api="blas"):
                sec1 = timed(lambda: ref.block_forward(x, W, "layers.0", d, ang, c), min_s=1.0)
            out[name + "_1thread"] = {"ms": sec1 * 1e3, "gflops": fl / sec1 / 1e9, "threads": 1,
                                      "speedup_all_threads": sec1 / sec}
    rate = out["block_4128"]["gflops"] * 1e9
    full = forward_flops(d, (LAT_H // 2) * (LAT_W // 2), S_TXT)
    out["full_forward_4128_extrapolated_s"] = full / rate
    print(json.dumps(out), flush=True)


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    step, flops, sample = oracle_sample()
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": value / (forward_flops(zi.FULL, (LAT_H // 2) * (LAT_W // 2), S_TXT) / PAGES_FORWARD_S / 1e12),
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": (LAT_H // 2) * (LAT_W // 2) + S_TXT, "batch": 1,
                   "sample_per_step": sample, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def make_fetch(d: zi.Dims, rank: int, world: int, device, threads: int):
    """fetch(keys) -> {key: bf16 bits}: rank 0 draws the seeded weights on its host
    threads and broadcasts them (over the process group's backend) to the other
    ranks, so every replica holds identical weights and the host draws them once."""
    import torch
    import torch.distributed as dist

    specs = {k: s for k, s, _ in zi.weight_specs(d)}

    def fetch(keys):
        out = zi.make_weights(d, seed=SEED, keys=keys, threads=threads) if rank == 0 or world == 1 else {}
        if world == 1:
            return out
        res = {}
        for k in keys:  # as raw bytes: neither NCCL nor gloo reduces or broadcasts 16-bit integers
            n = int(np.prod(specs[k])) * 2
            t = (torch.from_numpy(np.ascontiguousarray(out[k]).reshape(-1).view(np.uint8)).to(device) if rank == 0
                 else torch.empty(n, dtype=torch.uint8, device=device))
            dist.broadcast(t, 0)
            res[k] = t.cpu().numpy().view(np.uint16).reshape(specs[k])
        return res

    return fetch


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (each rank timed its own device)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from stream_diffusion_transformer_b200 import abi, model

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    d = zi.FULL
    cfg = model.make_config(d)
    s_img = (LAT_H // 2) * (LAT_W // 2)
    S = s_img + S_TXT
    flops = forward_flops(d, s_img, S_TXT)
    abi.clear_device_status()

    # weights: generated on rank 0's host threads, broadcast to the other ranks
    threads = max(1, min(32, (os.cpu_count() or 8)))

    fetch = make_fetch(d, rank, world, dev, threads)

    t_load = time.perf_counter()
    dit = model.DiT(cfg, fetch, device=dev)
    load_s = time.perf_counter() - t_load

    lat = torch.from_numpy(zi.make_latent(d, 1, LAT_H, LAT_W, seed=SEED)).to(dev)
    txt = torch.from_numpy(zi.make_text(d, 1, S_TXT, seed=SEED).view(np.int16)).to(dev).view(torch.bfloat16)
    tt = torch.full((1,), T_VALUE, dtype=torch.float32, device=dev)
    out = torch.empty_like(lat)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        dit.forward(lat, tt, txt, out)
    torch.cuda.synchronize()

    # ---- timed region: K forwards, inputs resident in HBM (no per-kernel events inside)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            dit.forward(lat, tt, txt, out)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    status = abi.device_status()
    if status != 0:
        raise RuntimeError(f"device pipeline timeout (code {status}) during the timed region")
    out_finite = bool(torch.isfinite(out).all().item())

    # ---- the same K forwards again with a CUDA event around every kernel launch
    # (per-kernel durations and rooflines; not part of the timed region above)
    with abi.Profile(capacity=600 * args.steps + 64) as prof:
        for _ in range(args.steps):
            dit.forward(lat, tt, txt, out)
        torch.cuda.synchronize()

    # ---- end to end through the public API: pinned host inputs in, result out, every step
    h_lat = torch.from_numpy(zi.make_latent(d, 1, LAT_H, LAT_W, seed=SEED)).pin_memory()
    h_txt = torch.from_numpy(zi.make_text(d, 1, S_TXT, seed=SEED).view(np.int16)).pin_memory()
    h_t = torch.full((1,), T_VALUE, dtype=torch.float32).pin_memory()
    h_out = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    d_lat, d_txt, d_t = torch.empty_like(lat), torch.empty(txt.shape, dtype=torch.int16, device=dev), torch.empty_like(tt)

    def e2e_step():
        d_lat.copy_(h_lat, non_blocking=True)
        d_txt.copy_(h_txt, non_blocking=True)
        d_t.copy_(h_t, non_blocking=True)
        dit.forward(d_lat, d_t, d_txt.view(torch.bfloat16), out)
        h_out.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    h2d = h_lat.numel() * 4 + h_txt.numel() * 2 + h_t.numel() * 4
    d2h = h_out.numel() * 4

    # ---- the same forward with e4m3 block projections (the quantised variants the pages
    # are about), on the resident bf16 weights: same inputs, same timing rules
    e4m3 = {}
    if not args.no_e4m3:
        for mode, name, what in ((True, "e4m3_qkv_ffn_up", "e4m3 QKV and FFN w1|w3 projections, bf16 elsewhere"),
                                 ("all", "e4m3_all_projections", "e4m3 QKV, output, FFN w1|w3 and w2 projections")):
            dit8 = dit.with_e4m3(mode)
            for _ in range(args.warmup):
                dit8.forward(lat, tt, txt, out)
            torch.cuda.synchronize()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(local_rank) as clk8:
                barrier()
                torch.cuda.synchronize()
                f0.record(stream)
                for _ in range(args.steps):
                    dit8.forward(lat, tt, txt, out)
                f1.record(stream)
                torch.cuda.synchronize()
                barrier()
            ms8 = max_over_ranks(f0.elapsed_time(f1), world, dev)
            e4m3[name] = {"value": flops * world * args.steps / (ms8 * 1e-3) / 1e12, "unit": "TFLOP/s",
                          "ms_per_step": ms8 / args.steps, "steps": args.steps, "warmup": args.warmup,
                          "dtype": what, "flops": "counted as for the bf16 forward",
                          "output_finite": bool(torch.isfinite(out).all().item()), "clocks": clk8.summary()}
            del dit8
            torch.cuda.empty_cache()
        if abi.device_status() != 0:
            raise RuntimeError("device pipeline timeout during the e4m3 forwards")

    # ---- the other two workloads of the pages on the same resident weights: the 8-step
    # Turbo loop (1024x1024 + 128 text tokens, replayed as one CUDA graph) and one CFG step
    # (2048x2048, batch 2 x (16,384 + 512) tokens, guidance 4); same timing rules, fewer steps
    workloads = {}
    if not args.no_workloads:
        def timed_extra(fn, n):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(local_rank) as clk_w:
                barrier()
                torch.cuda.synchronize()
                g0.record(stream)
                for _ in range(n):
                    fn()
                g1.record(stream)
                torch.cuda.synchronize()
                barrier()
            return max_over_ranks(g0.elapsed_time(g1), world, dev) / n, clk_w.summary()

        n_x = max(1, min(args.steps, 5))
        txt128 = torch.from_numpy(zi.make_text(d, 1, 128, seed=SEED).view(np.int16)).to(dev).view(torch.bfloat16)
        graph = model.DenoiseGraph(dit, tuple(lat.shape), txt128, n_steps=8)
        loop_ms, clk_l = timed_extra(lambda: graph.run(lat), n_x)
        loop_fl = 8 * forward_flops(d, s_img, 128)
        workloads["turbo8"] = {"what": f"8-step Turbo loop (shift 3), 1024x1024, {s_img} + 128 tokens, one CUDA graph "
                                       "(8 forwards and 8 Euler steps)",
                               "ms_per_loop": loop_ms, "ms_per_forward": loop_ms / 8,
                               "value": loop_fl * world / (loop_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                               "steps": n_x, "warmup": args.warmup,
                               "output_finite": bool(torch.isfinite(graph.out).all().item()), "clocks": clk_l}
        del graph
        torch.cuda.empty_cache()
        c_hw, c_txt = 256, 512
        lat_c1 = torch.from_numpy(zi.make_latent(d, 1, c_hw, c_hw, seed=SEED)).to(dev)
        lat_c = torch.cat([lat_c1, lat_c1], 0).contiguous()
        txt_c = torch.cat([torch.from_numpy(zi.make_text(d, 1, c_txt, seed=SEED).view(np.int16)),
                           torch.from_numpy(zi.make_text(d, 1, c_txt, seed=SEED, uncond=True).view(np.int16))],
                          0).to(dev).view(torch.bfloat16).contiguous()
        tt_c = torch.full((2,), T_VALUE, dtype=torch.float32, device=dev)
        out_c = torch.empty_like(lat_c)
        x_c = lat_c1.clone()
        sig = abi.sigmas(8, 3.0)

        def cfg_step():
            dit.forward(lat_c, tt_c, txt_c, out_c)
            model.euler_step(x_c, out_c[:1], out_c[1:], 4.0, sig[0], sig[1])

        cfg_ms, clk_c = timed_extra(cfg_step, max(1, min(args.steps, 3)))
        cfg_fl = forward_flops(d, (c_hw // 2) ** 2, c_txt, batch=2)
        workloads["cfg"] = {"what": f"CFG step, 2048x2048, batch 2 x ({(c_hw // 2) ** 2} + {c_txt}) tokens, guidance 4 "
                                    "(one batch-2 forward and the guided Euler step)",
                            "ms_per_step": cfg_ms, "value": cfg_fl * world / (cfg_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                            "steps": max(1, min(args.steps, 3)), "warmup": args.warmup,
                            "output_finite": bool(torch.isfinite(x_c).all().item()), "clocks": clk_c}
        del lat_c, txt_c, out_c, x_c
        dit._ws.clear()
        torch.cuda.empty_cache()
        if abi.device_status() != 0:
            raise RuntimeError("device pipeline timeout during the Turbo loop or the CFG step")

    if rank != 0:
        return

    # ---- per-kernel durations from the events recorded between launches in the timed region
    per_step = len(prof.kinds) // args.steps
    table = {}
    for k, m in zip(prof.kinds, prof.ms):
        e = table.setdefault(k, {"launches": 0, "ms": 0.0})
        e["launches"] += 1
        e["ms"] += m
    total_ms = sum(prof.ms)
    for k in table:
        table[k]["share"] = table[k]["ms"] / total_ms
        table[k]["ms_per_launch"] = table[k]["ms"] / table[k]["launches"]

    def main_block_launches(kind):
        """Durations of `kind` in the 30 main blocks (4,128 rows), per forward in launch order."""
        out_ms = []
        for sidx in range(args.steps):
            seq = [(k, m) for k, m in zip(prof.kinds[sidx * per_step:(sidx + 1) * per_step],
                                          prof.ms[sidx * per_step:(sidx + 1) * per_step]) if k == kind]
            out_ms += [m for _, m in seq[-d.n_main:]]
        return out_ms

    peaks, peak_src = load_peaks()
    peak_tensor = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    ffn_ms = statistics.mean(main_block_launches("gemm_ffn_up_swiglu"))
    ffn_flops = 2.0 * S * d.dim * (2 * d.ffn)
    ffn_tflops = ffn_flops / (ffn_ms * 1e-3) / 1e12
    att_ms = statistics.mean(main_block_launches("attention"))
    att_tflops = 4.0 * S * S * d.dim / (att_ms * 1e-3) / 1e12
    per_kernel_roof = {}
    for kind, fl in (("gemm_qkv_qknorm_rope", 6.0 * S * d.dim ** 2), ("attention", 4.0 * S * S * d.dim),
                     ("gemm_out_proj", 2.0 * S * d.dim ** 2), ("gemm_ffn_up_swiglu", ffn_flops),
                     ("gemm_ffn_down", 2.0 * S * d.dim * d.ffn)):
        m = statistics.mean(main_block_launches(kind))
        per_kernel_roof[kind] = {"ms_per_launch": m, "tflops": fl / (m * 1e-3) / 1e12,
                                 "frac": fl / (m * 1e-3) / 1e12 / peak_tensor, "traffic": recorded_traffic(kind)}
    for kind, bytes_per_row in (("post_norm_residual", 4 * d.dim * 2 + 2 * d.dim * 2),):
        m = statistics.mean(main_block_launches(kind))
        gbs = bytes_per_row * S / (m * 1e-3) / 1e9
        per_kernel_roof[kind] = {"ms_per_launch": m, "gbs": gbs, "frac": gbs / float(peaks["hbm_gbs"]),
                                 "algorithmic_bytes_per_launch": bytes_per_row * S, "traffic": recorded_traffic(kind)}

    clk = clocks.summary()
    sm_hz = float((clk or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)) * 1e6
    mufu_ms = d.heads * S * S / (16.0 * 148 * sm_hz) * 1e3
    value = flops * world * args.steps / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": value / (flops / PAGES_FORWARD_S / 1e12),
        "vs_baseline_note": "value / (55.12 TFLOP / 22.5 s): the pages' M1 Pro int8 forward of the same 4,128 tokens",
        "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": WORKLOAD, "tokens": S, "batch": 1, "image": "1024x1024", "text_tokens": S_TXT,
            "t": T_VALUE, "params": sum(int(np.prod(s)) for _, s, _ in zi.weight_specs(d)),
            "flops_per_step": flops, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "no flush: every step streams all 12.3 GB of weights (> 126 MB L2) from HBM",
            "cuda_graph": False, "weight_load_s": round(load_s, 1),
        },
        "tensor_peak_frac": value / world / peak_tensor,
        "roofline": {
            "kernel": "gemm_ffn_up_swiglu (main block, M=4128, N=20480, K=3840)",
            "bound": "tensor", "achieved": ffn_tflops, "peak": peak_tensor, "unit": "TFLOP/s",
            "frac": ffn_tflops / peak_tensor,
            "frac_of_burst": ffn_tflops / float(peaks["bf16_tflops"]),
            "spec_dense_peak": 2250.0,
            "traffic": recorded_traffic("gemm_ffn_up_swiglu"),
            "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
            "algorithmic_flops_per_launch": ffn_flops,
        },
        "attention_roofline": {"achieved": att_tflops, "peak": peak_tensor, "frac": att_tflops / peak_tensor,
                               "frac_of_burst": att_tflops / float(peaks["bf16_tflops"]),
                               "unit": "TFLOP/s", "ms_per_launch": att_ms,
                               # 30 S^2 exps at 16 per clock per SM (MUFU) at the measured median SM clock;
                               # the kernel moves 3 of 8 exps to the FMA pipe, so it can beat this bound
                               "mufu_exp_bound_ms": mufu_ms, "frac_of_mufu_bound": mufu_ms / att_ms},
        "kernels": {k: {kk: (round(vv, 5) if isinstance(vv, float) else vv) for kk, vv in e.items()}
                    for k, e in sorted(table.items(), key=lambda kv: -kv[1]["ms"])},
        "kernel_rooflines": per_kernel_roof,
        "gpu_launches": len(prof.kinds),
        "e2e": {"value": flops * world * args.steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / args.steps},
        "clocks": clk,
        "output_finite": out_finite,
        "e4m3_forwards": e4m3,
        "workloads": workloads,
        "published_context": {"ms": 22500.0, "hardware": "Apple M1 Pro", "precision": "int8 ConvRot",
                              "source": "Z-Image-Turbo repackaged for H3ddle, Measured performance"},
    }
    if world == 1 and not args.no_cpu_baseline:
        # the oracle's block, repeated until at least 10 s of CPU work (at most 4 runs)
        step, sflops, sample = oracle_sample()
        runs, t0 = 0, time.perf_counter()
        while runs < 4 and (runs == 0 or time.perf_counter() - t0 < 10.0):
            step()
            runs += 1
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": sflops * runs / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": f"{sample}, run {runs} times", "seconds": round(dt, 2)}
    print(json.dumps(line), flush=True)


def run_block_workload(args, fp8=False):
    """One full-width main block over the 4,128-token sequence (profiling-sized case, < 1 GB on the
    device); fp8 as for DeviceBlock (True: e4m3 QKV and FFN w1|w3, "all": every projection)."""
    import torch

    from stream_diffusion_transformer_b200 import abi, model

    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    cfg = model.make_config(d)
    gh, gw = LAT_H // 2, LAT_W // 2
    S = gh * gw + S_TXT
    bits = zi.make_weights(d, seed=SEED, keys=model.block_keys("layers.0", True), threads=8)
    blk = model.DeviceBlock(cfg, "layers.0", bits, True, "cuda", fp8=fp8)
    x = torch.from_numpy(zi.make_stream(d, 1, S, seed=SEED)).cuda()
    c = torch.from_numpy(zi.make_cond(d, 1, seed=SEED)).cuda()
    pos = model.positions(S_TXT, gh, gw)
    out = torch.empty_like(x)
    ws = torch.empty(abi.block_workspace_size(cfg, 1, S), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        model.block_forward(cfg, blk, c, pos, x, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with abi.Profile(capacity=16 * args.steps + 16) as prof:
        e0.record()
        for _ in range(args.steps):
            model.block_forward(cfg, blk, c, pos, x, out, ws)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    fl = block_flops(S, d.dim, d.ffn)
    tag = {False: "", True: ", e4m3 QKV and FFN w1|w3", "all": ", every projection in e4m3"}[fp8]
    print(json.dumps({"workload": f"one main block, full width, {S} tokens{tag}", "ms_per_step": ms,
                      "value": fl / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "steps": args.steps,
                      "kernels": prof.by_kernel(), "device_status": abi.device_status()}), flush=True)


def run_loop_workload(args, n_steps: int = 8, s_txt: int = 128):
    """The 8-step Turbo loop: 8 forwards at 4,096 image + 128 text tokens with the
    FlowMatch-Euler step (shift 3) between them; each timed step is one whole loop."""
    import torch

    from stream_diffusion_transformer_b200 import abi, model

    d = zi.FULL
    threads = max(1, min(32, (os.cpu_count() or 8)))
    dit = model.DiT(model.make_config(d), lambda keys: zi.make_weights(d, seed=SEED, keys=keys, threads=threads))
    lat = torch.from_numpy(zi.make_latent(d, 1, LAT_H, LAT_W, seed=SEED)).cuda()
    txt = torch.from_numpy(zi.make_text(d, 1, s_txt, seed=SEED).view(np.int16)).cuda().view(torch.bfloat16)
    graph = model.DenoiseGraph(dit, tuple(lat.shape), txt, n_steps=n_steps)  # the loop as one CUDA graph
    for _ in range(args.warmup):
        graph.run(lat)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        e0.record()
        for _ in range(args.steps):
            x = graph.run(lat)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    s_img = (LAT_H // 2) * (LAT_W // 2)
    fl = n_steps * forward_flops(d, s_img, s_txt)
    print(json.dumps({"workload": f"8-step Turbo loop, 1024x1024, {s_img} + {s_txt} tokens, shift 3, "
                                  "replayed as one CUDA graph",
                      "ms_per_loop": ms, "ms_per_forward": ms / n_steps, "value": fl / (ms * 1e-3) / 1e12,
                      "unit": "TFLOP/s", "steps": args.steps, "warmup": args.warmup,
                      "finite": bool(torch.isfinite(x).all().item()), "device_status": abi.device_status(),
                      "clocks": clocks.summary()}), flush=True)


def run_cfg_workload(args):
    """One classifier-free-guidance step at 2048x2048: a batch-2 forward (conditional
    and unconditional text, 16,384 image + 512 text tokens each) and the guidance-4
    combine inside the Euler update."""
    import torch

    from stream_diffusion_transformer_b200 import abi, model

    d = zi.FULL
    lat_hw, s_txt = 256, 512
    threads = max(1, min(32, (os.cpu_count() or 8)))
    dit = model.DiT(model.make_config(d), lambda keys: zi.make_weights(d, seed=SEED, keys=keys, threads=threads))
    lat1 = torch.from_numpy(zi.make_latent(d, 1, lat_hw, lat_hw, seed=SEED)).cuda()
    lat = torch.cat([lat1, lat1], 0).contiguous()
    txt = torch.cat([torch.from_numpy(zi.make_text(d, 1, s_txt, seed=SEED).view(np.int16)),
                     torch.from_numpy(zi.make_text(d, 1, s_txt, seed=SEED, uncond=True).view(np.int16))],
                    0).cuda().view(torch.bfloat16).contiguous()
    tt = torch.full((2,), T_VALUE, dtype=torch.float32, device="cuda")
    out = torch.empty_like(lat)
    x = lat1.clone()
    sig = abi.sigmas(8, 3.0)

    def step():
        dit.forward(lat, tt, txt, out)
        abi.call("zi_euler_step", model._p(x), model._p(out[:1]), model._p(out[1:]), 4.0, sig[0], sig[1],
                 x.numel(), model._stream())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks, abi.Profile(capacity=400 * args.steps + 16) as prof:
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    s_img = (lat_hw // 2) ** 2
    fl = forward_flops(d, s_img, s_txt, batch=2)
    by = {k: {"launches": v[0], "ms": round(v[1] / args.steps, 3)} for k, v in prof.by_kernel().items()}
    print(json.dumps({"workload": f"CFG step, 2048x2048, batch 2 x ({s_img} + {s_txt}) tokens, guidance 4",
                      "ms_per_step": ms, "value": fl / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "flops_per_step": fl, "steps": args.steps, "warmup": args.warmup, "kernels_ms_per_step": by,
                      "finite": bool(torch.isfinite(x).all().item()), "device_status": abi.device_status(),
                      "clocks": clocks.summary()}), flush=True)


def run_fp8_workload(args, mode=True):
    """The metric's forward (4,128 tokens at 1024x1024, batch 1) with every block's QKV
    and FFN w1|w3 projections in e4m3 (per-row scales, tcgen05 kind::f8f6f4); the other
    steps stay as in the bf16 forward.  FLOPs are counted as for the bf16 forward."""
    import torch

    from stream_diffusion_transformer_b200 import abi, model

    d = zi.FULL
    threads = max(1, min(32, (os.cpu_count() or 8)))
    dit = model.DiT(model.make_config(d), lambda keys: zi.make_weights(d, seed=SEED, keys=keys, threads=threads),
                    fp8=mode)
    lat = torch.from_numpy(zi.make_latent(d, 1, LAT_H, LAT_W, seed=SEED)).cuda()
    txt = torch.from_numpy(zi.make_text(d, 1, S_TXT, seed=SEED).view(np.int16)).cuda().view(torch.bfloat16)
    tt = torch.full((1,), T_VALUE, dtype=torch.float32, device="cuda")
    out = torch.empty_like(lat)
    for _ in range(args.warmup):
        dit.forward(lat, tt, txt, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks, abi.Profile(capacity=400 * args.steps + 16) as prof:
        e0.record()
        for _ in range(args.steps):
            dit.forward(lat, tt, txt, out)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    s_img = (LAT_H // 2) * (LAT_W // 2)
    S = s_img + S_TXT
    fl = forward_flops(d, s_img, S_TXT)
    peaks, peak_src = load_peaks()
    peak_f8 = 2.0 * float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))  # e4m3 = 2x bf16 (nominal ratio)
    per_step = len(prof.kinds) // args.steps
    roof = {}
    kinds = [("gemm_qkv_qknorm_rope", 6.0 * S * d.dim ** 2), ("gemm_ffn_up_swiglu", 4.0 * S * d.dim * d.ffn)]
    if mode == "all":
        kinds += [("gemm_out_proj", 2.0 * S * d.dim ** 2), ("gemm_ffn_down", 2.0 * S * d.dim * d.ffn)]
    for kind, kfl in kinds:
        ms_k = []
        for sidx in range(args.steps):
            seq = [m for k, m in zip(prof.kinds[sidx * per_step:(sidx + 1) * per_step],
                                     prof.ms[sidx * per_step:(sidx + 1) * per_step]) if k == kind]
            ms_k += seq[-d.n_main:]
        m = statistics.mean(ms_k)
        roof[kind] = {"ms_per_launch": m, "tflops": kfl / (m * 1e-3) / 1e12, "peak": peak_f8,
                      "frac": kfl / (m * 1e-3) / 1e12 / peak_f8,
                      "peak_source": f"{peak_src} bf16 sustained x 2 (nominal e4m3 / bf16 ratio)"}
    by = {k: {"launches": v[0], "ms": round(v[1] / args.steps, 3)} for k, v in prof.by_kernel().items()}
    what = "every block projection" if mode == "all" else "QKV + FFN-up projections"
    print(json.dumps({"workload": f"e4m3 {what}, 1024x1024, {s_img} + {S_TXT} tokens, batch 1",
                      "ms_per_step": ms, "value": fl / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "dtype": "e4m3 (all block projections) + bf16" if mode == "all" else "e4m3 (QKV, FFN w1|w3) + bf16",
                      "flops_per_step": fl, "steps": args.steps,
                      "warmup": args.warmup, "kernel_rooflines": roof, "kernels_ms_per_step": by,
                      "finite": bool(torch.isfinite(out).all().item()), "device_status": abi.device_status(),
                      "clocks": clocks.summary()}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e4m3", action="store_true", help="skip the e4m3 forwards after the headline timing")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the Turbo loop and the CFG step after the headline timing")
    ap.add_argument("--workload", choices=["forward", "block", "block8", "block8all", "turbo8", "cfg", "fp8", "fp8all",
                                           "oracle"], default="forward",
                    help="forward: the 4,128-token full forward (the metric); block: one main block of it "
                         "(a profiling-sized case; block8 / block8all: with e4m3 projections); turbo8: the 8-step denoising loop at 4,224 tokens; "
                         "cfg: one guidance step at 2048x2048, batch 2 x 16,896 tokens; fp8 / fp8all: the "
                         "forward with e4m3 projections; oracle: CPU oracle timings on this host")
    args = ap.parse_args()
    if args.workload == "oracle":
        run_oracle_workload(args)
        return
    if args.workload in ("block", "block8", "block8all"):
        run_block_workload(args, {"block": False, "block8": True, "block8all": "all"}[args.workload])
        return
    if args.workload == "turbo8":
        run_loop_workload(args)
        return
    if args.workload == "cfg":
        run_cfg_workload(args)
        return
    if args.workload in ("fp8", "fp8all"):
        run_fp8_workload(args, "all" if args.workload == "fp8all" else True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
