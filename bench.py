#!/usr/bin/env python
"""Benchmark of the MuScriptor KV-cached INT4 decoder step on B200.

One step = one pass of the whole decoder path over one synthetic input: reset the cache,
prefill [prefix (503 rows) ; start token] (504 positions), then greedy decode
(argmax fed back) for the workload's number of steps, through the library's C ABI
(ms_prefill + ms_generate).  Default workload: the medium shape (24 layers, d 1024, 16
heads with 4 kv heads, d_ff 4096, INT4 g32 backbone), batch 1, 2000 decode steps in a
2504-position cache.  Weights and inputs are seeded synthetic draws (synth module).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent replica on
its own GPU (the decoder does not shard); `value` sums all ranks' tokens over the slowest
rank's time.  `--impl reference` times the CPU oracle on this host's cores instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "decode ms/token & tokens/s (b=1, batched), prefill ms; % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="c3", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="override the workload's decode steps (short runs for profiling)")
    ap.add_argument("--cpu-decode-steps", type=int, default=256,
                    help="decode steps in the oracle's timed sample")
    ap.add_argument("--no-batched", action="store_true",
                    help="skip the batched-decode block (the 64-stream medium workload)")
    ap.add_argument("--no-prefill-tensor", action="store_true",
                    help="skip the prefill GEMM tensor-pipe block")
    ap.add_argument("--no-cond", action="store_true", help="skip the conditioner block")
    ap.add_argument("--no-w4a8", action="store_true", help="skip the W4A8 block")
    ap.add_argument("--no-pages", action="store_true",
                    help="skip the page-faithful block (kv heads = heads, fp32 and fp16 caches)")
    ap.add_argument("--decode-path", type=int, default=0, choices=[0, 1, 2],
                    help="0 automatic, 1 persistent decode kernel, 2 one kernel per operation")
    return ap.parse_args()


FALLBACK_BF16_TFLOPS = 1590.0
# Arithmetic each path runs (the weights are INT4 codes times fp32 group scales, or halves):
DTYPE = ("f32: fp32 activations, KV cache, LayerNorm, softmax and LM head; batch-1..8 decode "
         "matrix products on warp MMAs with each activation as an exact fp16 hi+lo pair (22-bit "
         "significand) and fp32 accumulation; prefill and batched-decode GEMMs on tcgen05 kind::f16 "
         "with both operands as fp16 hi+lo pairs (three products) and fp32 accumulation")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def _config_json(wl: synth.Workload, world: int):
    sh = wl.shape
    return {
        "workload": (f"{wl.name}: L{sh.n_layers} d{sh.d_model} H{sh.n_heads}/Hk{sh.n_kv_heads} F{sh.d_ff} "
                     f"V{sh.vocab} {wl.weight_format} backbone, batch {wl.batch}, prefill {wl.prefix_len}+1, "
                     f"{wl.decode_steps} greedy decode steps, cache {wl.capacity}"),
        "batch_per_gpu": wl.batch,
        "prefill_rows": wl.prefix_len + 1,
        "decode_steps": wl.decode_steps,
        "cache_capacity": wl.capacity,
        "l2": "weights+cache larger than L2; L2 flushed (256 MiB write) before every timed step",
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


# DRAM traffic of one launch of the persistent decode kernel, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; medium INT4 model, batch 1, the launch of
# decode steps 897..1024, cache lengths 1401..1528), with the kernel source it was taken on.
# A changed kernel source invalidates it (traffic is then reported as null).
_TRAFFIC = {
    "c3": {"bytes": 31.064088e9 + 15.687424e6, "tokens": 128, "T": (1401, 1528),
           "kernel_sha256_16": "15582d3ff2550257"},
}


def _kernel_sha16():
    import hashlib
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "decoder_only_transformer_int4_b200", "csrc",
                        "k_decode_persistent.cu")
    try:
        with open(path, "rb") as f:
            return hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None


def _decode_bytes_per_token(wl: synth.Workload, kv_elem: int = 4):
    """Algorithmic bytes of one decode step per stream set: backbone weights (+ scales for
    INT4), LM head, one embedding row per stream, and K and V over every cached position
    (kv_elem bytes per cache element: 4 for fp32, 2 for the half-precision cache).
    Returns (weight bytes per step, list of KV bytes per step over the run)."""
    sh = wl.shape
    w = 0
    for (n, k) in sh.matmul_shapes():
        w += n * k // 2 + n * (k // 32) * 4 if wl.weight_format == "int4" else n * k * 2
    w *= sh.n_layers
    w += sh.vocab * sh.d_model * 4 + wl.batch * sh.d_model * 4
    p0 = wl.prefix_len + 1
    kv = [2 * sh.n_layers * wl.batch * sh.n_kv_heads * (p0 + i + 1) * 64 * kv_elem for i in range(wl.decode_steps)]
    return w, kv


def _decode_bytes_at(wl: synth.Workload, T: int) -> float:
    """Algorithmic bytes of one decode step at cache length T (after its append)."""
    w, _ = _decode_bytes_per_token(dataclasses_replace_steps(wl, 0))
    sh = wl.shape
    return w + 2 * sh.n_layers * wl.batch * sh.n_kv_heads * T * 64 * 4


def dataclasses_replace_steps(wl: synth.Workload, steps: int) -> synth.Workload:
    import dataclasses
    return dataclasses.replace(wl, decode_steps=steps)


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sm)}


def _gpu_id(torch, dev: int) -> str:
    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


def _oracle_sample(wl: synth.Workload, n_decode: int):
    """Time the CPU oracle on a bounded sample of the workload: prefill of stream 0 and
    n_decode greedy steps.  Returns (tokens/s, seconds, threads, sample description)."""
    from oracle import ms_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    draw = synth.make_weights(wl.shape, seed=0)
    om = O.OracleModel(draw, wl.weight_format)
    prefix = synth.make_prefix(wl.shape, 1, wl.prefix_len, seed=1)[0]
    start = int(synth.make_start_tokens(1, seed=2)[0])
    t0 = time.perf_counter()
    om.greedy(prefix, start, n_decode, capacity=wl.prefix_len + 1 + n_decode)
    dt = time.perf_counter() - t0
    sample = (f"oracle (numpy fp64) on stream 0: prefill {wl.prefix_len}+1 rows then {n_decode} greedy "
              f"decode steps; tokens/s = {n_decode + 1} tokens / time")
    return (n_decode + 1) / dt, dt, threads, sample, om, draw


def max_over_ranks(x: float, device=None) -> float:
    """The largest x over all ranks of the job (the job takes as long as its slowest rank);
    x itself without a process group or with one rank."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step_per_rank: int, steps: int, world: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank (one replica per GPU) generates the same tokens per
    step; the time is the slowest rank's."""
    return world * tokens_per_step_per_rank * steps / (total_ms / 1e3)


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = synth.WORKLOADS[a.workload]
    from oracle import ms_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    draw = synth.make_weights(wl.shape, seed=0)
    om = O.OracleModel(draw, wl.weight_format)
    prefix = synth.make_prefix(wl.shape, 1, wl.prefix_len, seed=1)[0]
    start = int(synth.make_start_tokens(1, seed=2)[0])
    n_dec = a.cpu_decode_steps
    times = []
    for i in range(a.warmup + a.steps):
        t0 = time.perf_counter()
        om.greedy(prefix, start, n_dec, capacity=wl.prefix_len + 1 + n_dec)
        if i >= a.warmup:
            times.append(time.perf_counter() - t0)
    step = statistics.mean(times)
    value = (n_dec + 1) * wl.batch / step if wl.batch == 1 else (n_dec + 1) / step
    sample = (f"each step: oracle prefill {wl.prefix_len}+1 rows and {n_dec} greedy decode steps of stream 0 "
              f"(a bounded sample of the workload)")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": _config_json(wl, 1),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# The batched-decode workload that goes with each batch-1 workload (same model and weights).
_BATCHED = {"c3": "c4", "c5": "c5b16"}


def _batched_block(ms, torch, model, key, dev, flush, steps=2, warmup=1):
    """The batched half of the metric: the same model decoding many independent streams
    (prefill all, then greedy decode), device-timed like the main line.  Its roofline is the
    whole decode step's algorithmic bytes (weights + scales + LM head once, K and V of every
    stream) over the measured decode time."""
    wl = synth.WORKLOADS[key]
    sh, B = wl.shape, wl.batch
    stream = torch.cuda.current_stream(dev)
    prefix = torch.from_numpy(synth.make_prefix(sh, B, wl.prefix_len, seed=1)).to(dev)
    start = torch.from_numpy(synth.make_start_tokens(B, seed=2).reshape(B, 1)).to(dev)
    cache = ms.Cache(model, B, wl.capacity)
    out = torch.empty((wl.decode_steps, B), dtype=torch.int32, device=dev)

    def one(ev=None):
        cache.reset()
        flush.zero_()
        if ev:
            ev[0].record(stream)
        cache.prefill(start, prefix)
        if ev:
            ev[1].record(stream)
        cache.generate(wl.decode_steps, out_tokens=out, logits=False)
        if ev:
            ev[2].record(stream)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    l0 = cache.kernel_launches
    for i in range(steps):
        one(evs[i])
    torch.cuda.synchronize()
    launches = cache.kernel_launches - l0
    assert cache.device_status() == ms.MS_OK
    pre = [e[0].elapsed_time(e[1]) for e in evs]
    dec = [e[1].elapsed_time(e[2]) for e in evs]
    tot = [e[0].elapsed_time(e[2]) for e in evs]
    wbytes, kv = _decode_bytes_per_token(wl)
    dec_bytes = wbytes * wl.decode_steps + sum(kv)
    peak, kind = _peaks()
    ach = dec_bytes / (statistics.mean(dec) / 1e3) / 1e9
    path = cache.decode_path
    cache.close()
    return {
        "workload": _config_json(wl, 1)["workload"],
        "steps": steps, "warmup": warmup,
        "ms_per_step": statistics.mean(tot),
        "tokens_per_s": B * (wl.decode_steps + 1) / (statistics.mean(tot) / 1e3),
        "decode_ms_per_step": statistics.mean(dec) / wl.decode_steps,
        "decode_tokens_per_s": B * wl.decode_steps / (statistics.mean(dec) / 1e3),
        "prefill_ms": statistics.mean(pre),
        "decode_path": "persistent kernel" if path == 1 else "one kernel per operation, CUDA graph per step",
        "gpu_launches": launches,
        "roofline": {"bound": "hbm", "kernel": "decode step (all kernels of one step over every stream)",
                     "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak, "peak_kind": kind,
                     "algorithmic_bytes_per_step": dec_bytes / wl.decode_steps, "traffic": None},
    }


def _w4a8_block(ms, torch, model, wl, dev, flush, steps=2, warmup=1, decode_steps=256):
    """The W4A8 option (INT8 dynamic activation codes per 32-element block, dp4a integer dot
    products) on the benchmark's model and batch: prefill and a run of greedy decode steps on
    the per-operation path (the persistent kernel keeps fp32-level activations), device-timed
    with CUDA events, L2 flushed before each step.  Decode is timed alongside the fp32-activation
    run of the same path for comparison."""
    B, sh = wl.batch, wl.shape
    prefix = torch.from_numpy(synth.make_prefix(sh, B, wl.prefix_len, seed=1)).to(dev)
    start = torch.from_numpy(synth.make_start_tokens(B, seed=2).reshape(B, 1)).to(dev)
    out = torch.empty((decode_steps, B), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {"workload": f"{_config_json(wl, 1)['workload']}; {decode_steps} decode steps per timing",
           "decode_path": "one kernel per operation, CUDA graph per step"}
    for name, a8 in (("w4a8", True), ("w4a32", False)):
        cache = ms.Cache(model, B, wl.capacity)
        cache.set_decode_path(2)
        cache.set_act_int8(a8)
        pre, dec = [], []
        for i in range(warmup + steps):
            cache.reset()
            flush.zero_()
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            cache.prefill(start, prefix)
            e1.record(stream)
            cache.generate(decode_steps, out_tokens=out, logits=False)
            e2.record(stream)
            e2.synchronize()
            if i >= warmup:
                pre.append(e0.elapsed_time(e1))
                dec.append(e1.elapsed_time(e2))
        assert cache.device_status() == ms.MS_OK
        res[name] = {"prefill_ms": statistics.mean(pre), "decode_ms_per_step": statistics.mean(dec) / decode_steps,
                     "decode_tokens_per_s": B * decode_steps / (statistics.mean(dec) / 1e3)}
        cache.close()
    return res


def _e2e_audio_block(ms, torch, cache, wl, dev, flush, start_h, out_tok, steps=2, warmup=1):
    """The pages' pipeline end to end through the public API: a 5-s 440 Hz clip (fp32 at 16 kHz)
    copied in from pinned host memory with its dataset and instrument ids, the conditioner (the
    stand-in buffers of synth.make_cond_weights) making the decoder's 501 + 1 + 1 prefix rows,
    prefill with the start token, the greedy decode, the tokens copied back; CUDA events around
    all of it, L2 flushed before each step."""
    B, sh = wl.batch, wl.shape
    if wl.prefix_len != 503:
        return None
    cond = ms.Conditioner.from_draw(synth.make_cond_weights(sh.d_model), synth.N_SAMPLES, synth.HOP, max_batch=B,
                                    device=dev.index or 0)
    audio_h = torch.from_numpy(synth.make_tone(B)).pin_memory()
    ds_h = torch.ones(B, dtype=torch.int32).pin_memory()
    inst_h = torch.zeros((B, 1), dtype=torch.int32).pin_memory()
    audio, ds, inst = audio_h.to(dev), ds_h.to(dev), inst_h.to(dev)
    start = start_h.to(dev)
    prefix = torch.empty((B, cond.rows(1), sh.d_model), dtype=torch.float32, device=dev)
    out_h = torch.empty((wl.decode_steps, B), dtype=torch.int32).pin_memory()
    am_h = torch.empty((B,), dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(warmup + steps):
        cache.reset()
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        audio.copy_(audio_h, non_blocking=True)
        ds.copy_(ds_h, non_blocking=True)
        inst.copy_(inst_h, non_blocking=True)
        start.copy_(start_h, non_blocking=True)
        cond(audio, ds, inst, out=prefix)
        _, am = cache.prefill(start, prefix)
        cache.generate(wl.decode_steps, out_tokens=out_tok, logits=False)
        am_h.copy_(am, non_blocking=True)
        out_h.copy_(out_tok, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    assert cond.device_status() == ms.MS_OK and cache.device_status() == ms.MS_OK
    cond.close()
    ms_step = statistics.mean(times)
    return {"value": B * (wl.decode_steps + 1) / (ms_step / 1e3), "unit": "tokens/s", "ms_per_step": ms_step,
            "steps": steps, "warmup": warmup,
            "h2d_bytes_per_step": audio_h.numel() * 4 + ds_h.numel() * 4 + inst_h.numel() * 4 + start_h.numel() * 8,
            "d2h_bytes_per_step": out_h.numel() * 4 + am_h.numel() * 4,
            "pipeline": "audio 5 s at 16 kHz -> conditioner -> prefill 503+1 -> greedy decode -> tokens"}


def _pages_block(ms, torch, dev, flush, steps=2, warmup=1):
    """The page-faithful medium shape (kv heads = heads = 16: the W4A32 page's 469.5 MiB
    cache at 2504 positions) at batch 1, the whole prefill + 2000-step greedy run, once with
    the pages' fp32 cache and once with the half-precision cache option.  Each line's roofline
    counts the cache at its own element size."""
    wl = synth.WORKLOADS["c3pages"]
    sh = wl.shape
    stream = torch.cuda.current_stream(dev)
    draw = synth.make_weights(sh, seed=0)
    model = ms.Model.from_draw(draw, wl.weight_format, device=dev.index or 0)
    del draw
    prefix = torch.from_numpy(synth.make_prefix(sh, 1, wl.prefix_len, seed=1)).to(dev)
    start = torch.from_numpy(synth.make_start_tokens(1, seed=2).reshape(1, 1)).to(dev)
    out = torch.empty((wl.decode_steps, 1), dtype=torch.int32, device=dev)
    peak, kind = _peaks()
    res = {"workload": _config_json(wl, 1)["workload"], "steps": steps, "warmup": warmup}
    for name, fmt, es in (("kv_f32", ms.MS_KV_F32, 4), ("kv_f16", ms.MS_KV_F16, 2)):
        cache = ms.Cache(model, 1, wl.capacity, kv_format=fmt)
        dec = []
        for i in range(warmup + steps):
            cache.reset()
            flush.zero_()
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            cache.prefill(start, prefix)
            e1.record(stream)
            cache.generate(wl.decode_steps, out_tokens=out, logits=False)
            e2.record(stream)
            e2.synchronize()
            if i >= warmup:
                dec.append(e1.elapsed_time(e2))
        assert cache.device_status() == ms.MS_OK
        wbytes, kv = _decode_bytes_per_token(wl, es)
        tot = wbytes * wl.decode_steps + sum(kv)
        ach = tot / (statistics.mean(dec) / 1e3) / 1e9
        res[name] = {"decode_ms_per_token": statistics.mean(dec) / wl.decode_steps,
                     "decode_tokens_per_s": wl.decode_steps / (statistics.mean(dec) / 1e3),
                     "algorithmic_bytes_per_token": tot / wl.decode_steps,
                     "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                                  "peak_kind": kind}}
        cache.close()
    model.close()
    return res


# fp64 FMA lanes per SM on B200 (the published 37 TFLOP/s fp64 over 148 SMs at 1.965 GHz)
_FP64_LANES_PER_SM = 64


def _cond_block(ms, torch, dev, flush, d_model, batches, reps=5, warmup=2):
    """The conditioner front-end (5 s of 16 kHz audio -> 501 log-mel frames projected to
    d_model, then the dataset and instrument rows), device-timed per call with CUDA events, L2
    flushed before each.  The log-mel kernel alone is timed through ms_cond_log_mel (the same
    kernel writing fp32 rows instead of the GEMM's planes).  Its roofline is fp64 arithmetic:
    algorithmic flops per frame = 2.5 n log2 n for the real FFT of n = n_fft points, plus the
    window (n), the magnitudes (3 per bin) and the mel sums (2 per filterbank weight), against
    148 SMs x 64 fp64 FMA lanes x 2 flops x the SM clock (nominal, derived from unit counts)."""
    cond = synth.make_cond_weights(d_model)
    nnz = int((cond.mel_fb != 0).sum())
    n = synth.N_FFT
    flops_frame = 2.5 * n * math.log2(n) + n + 3 * (n // 2 + 1) + 2 * nnz
    props = torch.cuda.get_device_properties(dev)
    sm_ghz = 1.965
    peak64 = props.multi_processor_count * _FP64_LANES_PER_SM * 2 * sm_ghz * 1e9 / 1e12
    stream = torch.cuda.current_stream(dev)
    out = {"workload": f"conditioner: 5 s at 16 kHz (80000 samples), n_fft 2048, hop 160, 512 mel bands, "
                       f"d_model {d_model}, one instrument row", "cases": []}
    for B in batches:
        c = ms.Conditioner.from_draw(cond, synth.N_SAMPLES, synth.HOP, max_batch=B, device=dev.index or 0)
        audio = torch.from_numpy(synth.make_noise_audio(B, seed=6)).to(dev)
        dataset = torch.zeros(B, dtype=torch.int32, device=dev)
        inst = torch.zeros((B, 1), dtype=torch.int32, device=dev)
        prefix = torch.empty((B, c.rows(1), d_model), dtype=torch.float32, device=dev)
        lm = torch.empty((B, c.frames, synth.N_MELS), dtype=torch.float32, device=dev)
        t_all, t_lm = [], []
        for i in range(warmup + reps):
            for fn, acc in ((lambda: c(audio, dataset, inst, out=prefix), t_all), (lambda: c.log_mel(audio, out=lm), t_lm)):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                e1.synchronize()
                if i >= warmup:
                    acc.append(e0.elapsed_time(e1))
        assert c.device_status() == ms.MS_OK
        frames = B * c.frames
        ms_all, ms_lm = statistics.median(t_all), statistics.median(t_lm)
        ach = flops_frame * frames / (ms_lm / 1e3) / 1e12
        proj_tflop = 2.0 * frames * d_model * synth.N_MELS / 1e12
        out["cases"].append({
            "streams": B, "frames": frames, "ms_per_call": ms_all, "frames_per_s": frames / (ms_all / 1e3),
            "log_mel_ms": ms_lm, "projection_and_rows_ms": max(ms_all - ms_lm, 0.0),
            "projection_model_tflops": proj_tflop / (max(ms_all - ms_lm, 1e-6) / 1e3),
            "roofline": {"bound": "alu", "kernel": "log_mel_kernel (fp64 FFT, magnitudes, mel sums, log)",
                         "achieved": ach, "peak": peak64, "unit": "TFLOP/s", "frac": ach / peak64,
                         "peak_kind": f"derived: {props.multi_processor_count} SMs x {_FP64_LANES_PER_SM} fp64 "
                                      f"FMA lanes x 2 x {sm_ghz} GHz",
                         "algorithmic_flops_per_frame": flops_frame}})
        c.close()
    return out


def _prefill_tensor_block(ms, torch, model, shape, rows_list, dev, flush, reps=5, warmup=2):
    """Prefill GEMMs on the tensor cores: each backbone MatMul of layer 0 of the benchmark's
    model at M = prefill rows, through ms_model_matmul (the tcgen05 GEMM prefill runs, on the
    model's own tile-packed INT4 weights, from activation planes split beforehand),
    device-timed (CUDA events around each call, L2 flushed before each).  Model arithmetic is
    2 M N K per MatMul; the kernel issues three fp16 products per product (hi*hi, hi*lo,
    lo*hi), so its tensor issue rate is three times that, against the measured bf16 dense
    peak (fp16 and bf16 share the dense rate)."""
    bf16, kind = _bf16_peak()
    names = ["QKV", "O", "FC1", "FC2"]
    stream = torch.cuda.current_stream(dev)
    out = {"f16_peak_tflops": bf16, "f16_peak_derivation": f"{kind} bf16 dense {bf16:.1f} TFLOP/s (fp16 dense rate = bf16)",
           "issue_products_per_model_product": 3, "cases": []}
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    for M in rows_list:
        per, fl_tot, ms_tot = [], 0.0, 0.0
        for i, (name, (N, K)) in enumerate(zip(names, shape.matmul_shapes())):
            x = torch.randn(M, K, generator=g, dtype=torch.float32).to(dev)
            hi, lo = ms.split_f16(x)
            del x
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            times = []
            for it in range(warmup + reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                model.matmul(0, i, hi, lo, out=y)
                e1.record(stream)
                e1.synchronize()
                if it >= warmup:
                    times.append(e0.elapsed_time(e1))
            t = statistics.median(times)
            fl = 2.0 * M * N * K
            per.append({"matmul": name, "N": N, "K": K, "ms": t, "model_tflops": fl / t / 1e9,
                        "issue_tflops": 3 * fl / t / 1e9})
            fl_tot += fl
            ms_tot += t
            del hi, lo, y
        model_tf = fl_tot / ms_tot / 1e9
        out["cases"].append({"M": M, "matmuls": per, "layer_ms": ms_tot, "model_tflops": model_tf,
                             "issue_tflops": 3 * model_tf, "frac_of_f16_peak": 3 * model_tf / bf16})
    return out


def run_ours(a):
    import torch
    import torch.distributed as dist

    import decoder_only_transformer_int4_b200 as ms

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = synth.WORKLOADS[a.workload]
    if a.decode_steps is not None:
        import dataclasses
        wl = dataclasses.replace(wl, decode_steps=a.decode_steps)
    sh, B = wl.shape, wl.batch

    draw = synth.make_weights(sh, seed=0)
    model = ms.Model.from_draw(draw, wl.weight_format, device=local)
    del draw
    prefix_h = torch.from_numpy(synth.make_prefix(sh, B, wl.prefix_len, seed=1)).pin_memory()
    start_h = torch.from_numpy(synth.make_start_tokens(B, seed=2).reshape(B, 1)).pin_memory()
    prefix = prefix_h.to(dev)
    start = start_h.to(dev)
    cache = ms.Cache(model, B, wl.capacity)
    cache.set_decode_path(a.decode_path)
    out_tok = torch.empty((wl.decode_steps, B), dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2 ** 20 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one_step(e0=None, e1=None, e2=None):
        cache.reset()
        flush.zero_()
        if e0 is not None:
            e0.record(stream)
        cache.prefill(start, prefix)
        if e1 is not None:
            e1.record(stream)
        cache.generate(wl.decode_steps, out_tokens=out_tok, logits=False)
        if e2 is not None:
            e2.record(stream)

    for _ in range(a.warmup):
        one_step()
    torch.cuda.synchronize()
    assert cache.device_status() == ms.MS_OK

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(a.steps)]
    sampler = ClockSampler(_gpu_id(torch, local))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    launches0 = cache.kernel_launches
    t_wall = time.perf_counter()
    for i in range(a.steps):
        one_step(*ev[i])
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    launches = cache.kernel_launches - launches0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    assert cache.device_status() == ms.MS_OK

    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    pre_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    tokens_per_step = B * (wl.decode_steps + 1)
    value = job_throughput(tokens_per_step, a.steps, world, total_ms)
    per_tok = [d / wl.decode_steps for d in dec_ms]

    wbytes, kv = _decode_bytes_per_token(wl)
    dec_bytes = wbytes * wl.decode_steps + sum(kv)
    peak, peak_kind = _peaks()
    achieved = dec_bytes / (statistics.mean(dec_ms) / 1e3) / 1e9

    # end to end through host buffers: prefix and start token copied in from pinned host
    # memory, generated tokens copied back, every step.
    out_h = torch.empty((wl.decode_steps, B), dtype=torch.int32).pin_memory()
    am_h = torch.empty((B,), dtype=torch.int32).pin_memory()
    e2e_ms = []
    for i in range(0 if a.no_e2e else max(1, min(a.steps, 3))):
        cache.reset()
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        prefix.copy_(prefix_h, non_blocking=True)
        start.copy_(start_h, non_blocking=True)
        _, am = cache.prefill(start, prefix)
        cache.generate(wl.decode_steps, out_tokens=out_tok, logits=False)
        am_h.copy_(am, non_blocking=True)
        out_h.copy_(out_tok, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    h2d = prefix_h.numel() * 4 + start_h.numel() * 8
    d2h = out_h.numel() * 4 + am_h.numel() * 4
    # every rank ran the same e2e steps, so every rank takes part in the reduction
    e2e_job_ms = max_over_ranks(statistics.mean(e2e_ms), dev) if e2e_ms else None
    e2e_val = world * tokens_per_step / (e2e_job_ms / 1e3) if e2e_job_ms else None

    e2e_audio = None
    if world == 1 and not a.no_e2e:
        e2e_audio = _e2e_audio_block(ms, torch, cache, wl, dev, flush, start_h, out_tok)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, dt, threads, sample, _, _ = _oracle_sample(wl, a.cpu_decode_steps)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
               "seconds": dt}

    # roofline of the dominant kernel: the persistent decode kernel (one launch per 128 decode
    # steps, so per-launch figures are 128 x the per-token ones), else the per-operation graph
    persistent = cache.decode_path == 1
    roof = {"bound": "hbm",
            "kernel": ("decode_persistent_kernel (all layers, LM head and argmax of up to 128 decode steps "
                       "per launch)") if persistent else "decode step (all kernels of one token, one CUDA graph)",
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
            "traffic": None, "algorithmic_bytes_per_token": dec_bytes / wl.decode_steps}
    tr = _TRAFFIC.get(a.workload)
    if persistent and tr and tr["kernel_sha256_16"] == _kernel_sha16() and a.decode_steps is None:
        t_lo, t_hi = tr["T"]
        alg = sum(_decode_bytes_at(wl, t) for t in range(t_lo, t_hi + 1))
        roof["traffic"] = tr["bytes"]
        roof["traffic_per"] = f"one launch of {tr['tokens']} decode steps, cache lengths {t_lo}..{t_hi} (ncu)"
        roof["traffic_over_algorithmic"] = tr["bytes"] / alg
    batched = prefill_tc = pages = cond = w4a8 = None
    if world == 1 and not a.no_batched and a.workload in _BATCHED:
        batched = _batched_block(ms, torch, model, _BATCHED[a.workload], dev, flush)
    if world == 1 and not a.no_pages and a.workload == "c3":
        pages = _pages_block(ms, torch, dev, flush)
    if world == 1 and not a.no_prefill_tensor:
        rows = [wl.prefix_len + 1]
        if a.workload in _BATCHED:
            rows.append(synth.WORKLOADS[_BATCHED[a.workload]].batch * (wl.prefix_len + 1))
        prefill_tc = _prefill_tensor_block(ms, torch, model, sh, rows, dev, flush)
    if world == 1 and not a.no_w4a8 and sh.n_layers > 0 and wl.weight_format == "int4":
        w4a8 = _w4a8_block(ms, torch, model, wl, dev, flush)
    if world == 1 and not a.no_cond:
        nb = [1] + ([synth.WORKLOADS[_BATCHED[a.workload]].batch] if a.workload in _BATCHED else [])
        cond = _cond_block(ms, torch, dev, flush, sh.d_model, nb)
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": total_ms / a.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "data": "synthetic", "config": _config_json(wl, world),
            "prefill_ms": {"mean": statistics.mean(pre_ms), "median": statistics.median(pre_ms)},
            "decode_ms_per_token": {"mean": statistics.mean(per_tok), "median": statistics.median(per_tok),
                                    "p90": float(np.percentile(per_tok, 90))},
            "decode_tokens_per_s": B * wl.decode_steps / (statistics.mean(dec_ms) / 1e3),
            "roofline": roof,
            "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks,
            "wall_s": t_wall,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if batched is not None:
            line["batched"] = batched
        if prefill_tc is not None:
            line["prefill_tensor"] = prefill_tc
        if pages is not None:
            line["pages"] = pages
        if cond is not None:
            line["conditioner"] = cond
        if w4a8 is not None:
            line["w4a8"] = w4a8
        if e2e_audio is not None:
            line["e2e_audio"] = e2e_audio
        print(json.dumps(line), flush=True)
    cache.close()
    model.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
