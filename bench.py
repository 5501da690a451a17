#!/usr/bin/env python
"""Benchmark of the LLaMA decoder-block library on B200.

Default workload (one step): a LLaMA-1-7B-shaped decoder layer in bf16
(dim 4096, 32 heads, MHA, ffn 11008), batch 1: a 512-token prefill from
start_pos 0, then 128 single-token decode steps at positions 512..639, all
through llama_block_forward. The 128 decode steps of a pass are captured in
one CUDA graph together with the prefill; the graph also restores the step's
inputs first, so every step does identical work. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload llama7b-layer|llama70b-layer|llama3-8b-decode|llama3-8b-prefill]

With N > 1 (launched by torch.distributed.run) every rank runs an
independent replica (the workload has no exchange step); rank 0 prints the
aggregate over ranks, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from llama_decoder_block_kv_b200 import binding as B  # noqa: E402
from llama_decoder_block_kv_b200 import synth  # noqa: E402

METRIC = "prefill & decode tokens/s on 1 B200; % of HBM / bf16 tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


class NvmlClockSampler:
    """Read-only NVML sampling of the SM clock and the clock-event reasons every
    ~5 ms from a thread while the timed region runs (short regions still get
    samples; a final sample is taken at stop). Falls back to nvidia-smi."""
    REASONS = (("hw_slowdown", "nvmlClocksThrottleReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksThrottleReasonSwPowerCap", 0x4))

    def __init__(self, index: int):
        self.index = index
        self.fallback = None
        self.samples = []
        self.path = os.path.join(CLOCK_LOG_DIR, f"clocks_rank{index}.csv")
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_sm = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.bits = {n: getattr(pynvml, c, b) for n, c, b in self.REASONS}
        except Exception:
            self.nv = None
            self.fallback = ClockSampler(index)

    def _sample(self):
        nv = self.nv
        sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((time.time(), sm, int(r)))

    def _run(self):
        while not self.done.is_set():
            try:
                self._sample()
            except Exception:
                return
            self.done.wait(0.005)

    def start(self):
        if self.fallback is not None:
            return self.fallback.start()
        import threading
        self.done = threading.Event()
        self._sample()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.fallback is not None:
            return self.fallback.stop()
        self.done.set()
        self.thread.join(timeout=5)
        try:
            self._sample()
        except Exception:
            pass
        reasons = set()
        for _, _, r in self.samples:
            for n, b in self.bits.items():
                if r & b:
                    reasons.add(n)
        sm = [x[1] for x in self.samples]
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            with open(self.path, "w") as f:
                f.write("time,clocks.sm,clocks.max.sm,reasons_bits\n")
                for t, c, r in self.samples:
                    f.write(f"{t:.4f},{c:.0f},{self.max_sm:.0f},{r:#x}\n")
        except Exception:
            pass
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_sm, "samples": len(sm),
                "reasons": sorted(reasons), "source": "nvml"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(CLOCK_LOG_DIR, f"clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank takes part, rank order does not matter."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step_per_rank: int, steps: int, max_ms: float, world: int) -> float:
    """Whole-job tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step_per_rank * steps / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- single-layer workloads

class LayerBench:
    """Prefill + decode of one decoder layer (llama7b-layer) or decode only (llama70b-layer)."""

    def __init__(self, w: synth.Workload):
        self.w = w
        self.args = B.ModelArgs.from_workload(w)
        self.model = B.Llama(self.args)
        B.llama_set_decode_kernel(self.model.ctx, DECODE_KERNELS[DECODE_KERNEL])
        B.llama_set_decode_attention(self.model.ctx, DECODE_ATTENTIONS[DECODE_ATTENTION])
        self.lw = synth.layer_weights(w, 0, device="cuda")
        B.llama_set_layer(self.model.ctx, 0, self.lw)
        dim = w.dim
        self.P = w.prefill_len
        self.ND = w.decode_steps
        self.Bsz = w.batch
        if w.cache_len:  # decode-only workload with a prefilled cache
            shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
            k = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            v = torch.zeros_like(k)
            k[:, :w.cache_len] = synth.cache_values(w, 0, 0, (w.max_batch_size, w.cache_len, w.n_kv_heads,
                                                              w.head_dim), "cuda")
            v[:, :w.cache_len] = synth.cache_values(w, 0, 1, (w.max_batch_size, w.cache_len, w.n_kv_heads,
                                                              w.head_dim), "cuda")
            B.llama_kv_write(self.model.ctx, 0, k, v)
            del k, v
        self.dec_pos0 = w.cache_len if w.cache_len else self.P
        self.h_pre0 = synth.hidden(w, (self.Bsz, self.P, dim), 0, "cuda") if self.P else None
        self.h_dec0 = synth.hidden(w, (self.ND, self.Bsz, 1, dim), 1, "cuda")
        self.h_pre = self.h_pre0.clone() if self.P else None
        self.h_dec = self.h_dec0.clone()
        B.llama_reserve(self.model.ctx, max(self.Bsz * max(self.P, 1), 1))
        self.tokens_per_step = self.Bsz * (self.P + self.ND)
        self.graph = None

    def enqueue(self, phase="all"):
        ctx = self.model.ctx
        if self.P and phase in ("all", "prefill"):
            self.h_pre.copy_(self.h_pre0)
            B.llama_block_forward(ctx, 0, self.h_pre, 0)
        if phase in ("all", "decode"):
            self.h_dec.copy_(self.h_dec0)
            for i in range(self.ND):
                B.llama_block_forward(ctx, 0, self.h_dec[i], self.dec_pos0 + i)

    def capture(self, phase="all"):
        self.enqueue(phase)  # warm (function attributes, workspace) outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.enqueue(phase)
        torch.cuda.synchronize()
        return g

    def kernels_per_step(self):
        pre = 7 if self.P else 0  # rmsnorm, gemm x2, attention, rmsnorm, gemm x2 (the QKV and wo GEMMs: 4 in all)
        # decode: rmsnorm, gemv, attention (chunk merge fused), gemv, rmsnorm, gemv, gemv; or one persistent launch
        dec = 1 if DECODE_KERNEL == "persistent" else 7
        return pre + self.ND * dec

    def decode_gemms(self):
        """(x, w) pairs of the decode linears, same shapes and kernel as the decode path."""
        lw, w = self.lw, self.w
        M = self.Bsz
        wqkv = torch.cat([lw["wq"], lw["wk"], lw["wv"]], 0).contiguous()
        w13 = torch.stack([lw["w1"], lw["w3"]], 1).reshape(2 * w.ffn_hidden, w.dim).contiguous()
        xs = {K: synth.normal((M, K), 1.0, 7 + K, torch.bfloat16, "cuda") for K in (w.dim, w.ffn_hidden,
                                                                                  w.n_heads * w.head_dim)}
        return [(xs[w.dim], wqkv), (xs[w.n_heads * w.head_dim], lw["wo"]), (xs[w.dim], w13),
                (xs[w.ffn_hidden], lw["w2"])]

    def close(self):
        self.model.close()


def time_graph(g, steps, warmup, world):
    for _ in range(warmup):
        g.replay()
    barrier(world)
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        g.replay()
    e1.record(st)
    e1.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)


# DRAM traffic per algorithmic byte of the decode GEMV, from the committed ncu
# capture of one w1|w3 launch, M=1, N=22016, K=4096 (dram read + write of one
# launch / weights + activations + outputs). Valid for the kernel version that
# capture names; set to None when the kernel changes until it is re-measured.
GEMV_TRAFFIC_RATIO = (180.45e6 + 3.53e6) / (22016 * 4096 * 2 + 4096 * 2 + 22016 * 4)


def gemv_roofline(lb: LayerBench, peaks, reps=10):
    """Average bandwidth of the decode GEMV kernel: the layer's four decode linears
    (wqkv, wo, w1|w3, w2: 405 MB together, larger than L2) launched back to back
    `reps` times inside one CUDA graph, timed with CUDA events around the replay.
    Algorithmic bytes: weights + activations in + fp32 outputs."""
    pairs = lb.decode_gemms()
    ys = [torch.empty((x.shape[0], w.shape[0]), device="cuda") for x, w in pairs]
    byts = sum(w.numel() * 2 + x.numel() * 2 + x.shape[0] * w.shape[0] * 4 for x, w in pairs)
    # the weights in the tile layout the library keeps for its own linears
    tiles = [(x, B.llama_tile_weights(w), w.shape[0]) for x, w in pairs]
    path = B.LLAMA_PATH_GEMV | B.LLAMA_WEIGHTS_TILED
    for (x, wt, n), y in zip(tiles, ys):
        B.llama_linear(x, wt, y, path, n=n)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            for (x, wt, n), y in zip(tiles, ys):
                B.llama_linear(x, wt, y, path, n=n)
    g.replay()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    g.replay()
    e1.record(st)
    e1.synchronize()
    launches = reps * len(pairs)
    t_ms = e0.elapsed_time(e1) / launches          # average launch duration
    per_launch = byts / len(pairs)
    achieved = per_launch / (t_ms * 1e-3) / 1e9
    traffic = None if GEMV_TRAFFIC_RATIO is None else int(round(GEMV_TRAFFIC_RATIO * per_launch))
    return {"kernel": "gemv_bf16_kernel (decode linears: wqkv, wo, w1|w3, w2)", "bound": "hbm",
            "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
            "traffic_source": "ncu dram read+write of the w1|w3 launch scaled by algorithmic bytes "
                              "(M=1, N=22016, K=4096)",
            "bytes_per_launch": int(per_launch), "avg_launch_us": round(t_ms * 1e3, 2),
            "launches_timed": launches}


# ----------------------------------------------------------------------------- CPU oracle legs

def oracle_layer_sample(w: synth.Workload, n_decode: int = 4):
    """Time the oracle on one layer: the full prefill plus n_decode decode steps;
    returns (seconds for the workload's mix extrapolated from the sample, threads, sample text)."""
    import oracle as O

    def t2np(t):
        return t.detach().to("cpu", torch.float64).numpy()

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    lw = synth.layer_weights(w, 0)
    m = O.OracleModel(O.ModelArgs(dim=w.dim, n_layers=1, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                                  vocab_size=w.vocab_size, multiple_of=w.multiple_of,
                                  ffn_dim_multiplier=w.ffn_dim_multiplier, norm_eps=w.norm_eps,
                                  rope_theta=w.rope_theta, max_batch_size=w.max_batch_size,
                                  max_seq_len=w.max_seq_len, act=w.act))
    m.layers[0] = {k: t2np(v) for k, v in lw.items()}  # float64 weights, widened once
    if w.cache_len:
        m.cache_k[0][:, :w.cache_len] = t2np(synth.cache_values(w, 0, 0, (w.max_batch_size, w.cache_len,
                                                                         w.n_kv_heads, w.head_dim)))
        m.cache_v[0][:, :w.cache_len] = t2np(synth.cache_values(w, 0, 1, (w.max_batch_size, w.cache_len,
                                                                         w.n_kv_heads, w.head_dim)))
    t_pre = 0.0
    if w.prefill_len:
        h = t2np(synth.hidden(w, (w.batch, w.prefill_len, w.dim), 0))
        t0 = time.perf_counter()
        m.block(0, h, 0)
        t_pre = time.perf_counter() - t0
    pos0 = w.cache_len if w.cache_len else w.prefill_len
    hd = t2np(synth.hidden(w, (n_decode, w.batch, 1, w.dim), 1))
    t0 = time.perf_counter()
    for i in range(n_decode):
        m.block(0, hd[i], pos0 + i)
    t_dec = (time.perf_counter() - t0) / n_decode
    total = t_pre + w.decode_steps * t_dec
    sample = (f"oracle (numpy float64) on one layer: prefill of {w.prefill_len} tokens timed in full, "
              f"{n_decode} of {w.decode_steps} decode steps timed and extrapolated linearly")
    return total, threads, sample


# ----------------------------------------------------------------------------- main

def run_ours(args, world, rank, local):
    w = synth.WORKLOADS[args.workload]
    peaks, peak_kind = load_peaks()
    if w.n_layers > 1 and w.vocab_size > 0:
        return run_model_bench(args, world, rank, local, w, peaks, peak_kind)
    lb = LayerBench(w)
    g = lb.capture("all")
    sampler = NvmlClockSampler(local)
    barrier(world)
    sampler.start()
    ms = time_graph(g, args.steps, args.warmup, world)
    clocks = sampler.stop()
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = job_throughput(lb.tokens_per_step, args.steps, ms, world)

    # phases, each timed the same way
    phases = {}
    if lb.P:
        gp = lb.capture("prefill")
        tp = max_over_ranks(time_graph(gp, max(3, args.steps), args.warmup, world), world) / max(3, args.steps)
        flops = 2.0 * lb.P * lb.Bsz * (w.dim * (w.n_heads + 2 * w.n_kv_heads) * w.head_dim +
                                       w.n_heads * w.head_dim * w.dim + 3 * w.dim * w.ffn_hidden)
        flops += 4.0 * w.n_heads * w.head_dim * sum(s + 1 for s in range(lb.P)) * lb.Bsz
        phases["prefill_ms"] = round(tp, 4)
        phases["prefill_tok_s"] = round(world * lb.Bsz * lb.P / (tp * 1e-3), 1)
        phases["prefill_tflops"] = round(flops / (tp * 1e-3) / 1e12, 1)
        phases["prefill_tensor_frac"] = round(flops / (tp * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)
        del gp
    gd = lb.capture("decode")
    td = max_over_ranks(time_graph(gd, max(3, args.steps), args.warmup, world), world) / max(3, args.steps)
    wbytes = 2 * (w.dim * (w.n_heads + 2 * w.n_kv_heads) * w.head_dim + w.n_heads * w.head_dim * w.dim +
                  3 * w.dim * w.ffn_hidden)
    kvbytes = sum((lb.dec_pos0 + i + 1) * 2 * w.n_kv_heads * w.head_dim * 2 * lb.Bsz for i in range(lb.ND))
    phases["decode_ms_per_step"] = round(td / lb.ND, 5)
    phases["decode_tok_s"] = round(world * lb.Bsz * lb.ND / (td * 1e-3), 1)
    phases["decode_hbm_gbs"] = round((lb.ND * wbytes + kvbytes) / (td * 1e-3) / 1e9, 1)
    phases["decode_hbm_frac"] = round(phases["decode_hbm_gbs"] / peaks["hbm_gbs"], 4)
    del gd

    roof = gemv_roofline(lb, peaks)
    roof["peak_kind"] = peak_kind

    # end to end through the C ABI with host buffers: H2D of the step's inputs, D2H of its outputs
    e2e = run_e2e(lb, g, args, world)

    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic: seeded N(0,1) hidden states, N(0,0.02) weights, RMSNorm weights 1",
           "config": {"workload": w.name, "batch": lb.Bsz, "prefill_tokens": lb.P, "decode_steps": lb.ND,
                      "decode_start_pos": lb.dec_pos0, "l2": "inputs larger than L2: %.0f MB of weights per pass"
                      % (wbytes / 1e6), "parallelism": "replicas" if world > 1 else "single GPU",
                      "decode_kernel": DECODE_KERNEL, "decode_attention": DECODE_ATTENTION},
           "phases": phases, "roofline": roof, "e2e": e2e,
           "gpu_launches": lb.kernels_per_step() * args.steps, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, threads, sample = oracle_layer_sample(w)
        out["cpu_baseline"] = {"value": round(lb.tokens_per_step / t_cpu, 2), "unit": "tokens/s", "cores": threads,
                               "kind": "oracle", "sample": sample}
    lb.close()
    return out


def run_e2e(lb: LayerBench, g, args, world):
    """Same metric with host buffers: pinned H2D of inputs and D2H of outputs inside the timed region."""
    hin_pre = lb.h_pre0.cpu().pin_memory() if lb.P else None
    hin_dec = lb.h_dec0.cpu().pin_memory()
    hout_pre = torch.empty_like(hin_pre).pin_memory() if lb.P else None
    hout_dec = torch.empty_like(hin_dec).pin_memory()
    st = torch.cuda.current_stream()

    def step():
        if lb.P:
            lb.h_pre0.copy_(hin_pre, non_blocking=True)
        lb.h_dec0.copy_(hin_dec, non_blocking=True)
        g.replay()
        if lb.P:
            hout_pre.copy_(lb.h_pre, non_blocking=True)
        hout_dec.copy_(lb.h_dec, non_blocking=True)

    for _ in range(args.warmup):
        step()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    e1.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    bi = (hin_pre.numel() * 4 if lb.P else 0) + hin_dec.numel() * 4
    return {"value": round(world * lb.tokens_per_step * args.steps / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bi}


def run_model_bench(args, world, rank, local, w, peaks, peak_kind):
    """Whole-model workloads (LLaMA-3-8B shape): ragged decode or long prefill."""
    m = B.Llama(B.ModelArgs.from_workload(w))
    ctx = m.ctx
    B.llama_set_decode_kernel(ctx, DECODE_KERNELS[DECODE_KERNEL])
    B.llama_set_decode_attention(ctx, DECODE_ATTENTIONS[DECODE_ATTENTION])
    for i in range(w.n_layers):
        B.llama_set_layer(ctx, i, synth.layer_weights(w, i, device="cuda"))
    enh = synth.embed_norm_head(w, device="cuda")
    B.llama_set_embed_norm_head(ctx, enh["tok_embeddings"], enh["norm"], enh["output"])
    del enh
    if w.decode_steps:
        lens = synth.ragged_lengths(w, "cuda")
        shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
        for i in range(w.n_layers):
            k = synth.cache_values(w, i, 0, shape, "cuda")
            v = synth.cache_values(w, i, 1, shape, "cuda")
            B.llama_kv_write(ctx, i, k, v)
            del k, v
        toks = synth.tokens(w, (w.decode_steps, w.batch), 0, "cuda")
        pos = (lens[None, :] + torch.arange(w.decode_steps, device="cuda", dtype=torch.int32)[:, None]).contiguous()
        logits = torch.empty((w.batch, w.vocab_size), device="cuda")
        B.llama_reserve(ctx, w.batch)

        def enqueue():
            for s in range(w.decode_steps):
                B.llama_forward_ragged(ctx, toks[s], pos[s], logits)
        tokens_per_step = w.batch * w.decode_steps
        # per forward: embedding, the blocks, final RMSNorm, LM head
        per_block = 1 if DECODE_KERNEL == "persistent" else 7
        launches_per_step = w.decode_steps * (1 + w.n_layers * per_block + 2)
    else:
        toks = synth.tokens(w, (w.batch, w.prefill_len), 0, "cuda")
        logits = torch.empty((w.batch, w.vocab_size), device="cuda")
        B.llama_reserve(ctx, w.batch * w.prefill_len)

        def enqueue():
            B.llama_forward(ctx, toks, 0, logits, False)
        tokens_per_step = w.batch * w.prefill_len
        launches_per_step = 1 + w.n_layers * 7 + 2
    enqueue()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        enqueue()
    sampler = NvmlClockSampler(local)
    sampler.start()
    ms = max_over_ranks(time_graph(g, args.steps, args.warmup, world), world)
    clocks = sampler.stop()
    code, flags = B.llama_get_error(ctx)
    out = {"metric": METRIC, "value": round(world * tokens_per_step * args.steps / (ms * 1e-3), 1),
           "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": w.name, "decode_kernel": DECODE_KERNEL,
                                                "decode_attention": DECODE_ATTENTION}, "clocks": clocks, "device_error": code,
           "gpu_launches": launches_per_step * args.steps}
    m.close()
    return out


def run_reference(args, world, rank):
    """The oracle (CPU, numpy float64) as the reference arm, on rank 0 only."""
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    times = []
    threads, sample = None, None
    for i in range(args.warmup + args.steps):
        t, threads, sample = oracle_layer_sample(w, n_decode=2)
        if i >= args.warmup:
            times.append(t)
    t = sum(times) / len(times)
    value = (w.batch * (w.prefill_len + w.decode_steps)) / t
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


DECODE_KERNELS = {"auto": B.LLAMA_DECODE_AUTO, "layered": B.LLAMA_DECODE_LAYERED,
                  "persistent": B.LLAMA_DECODE_PERSISTENT}
DECODE_KERNEL = "auto"
DECODE_ATTENTIONS = {"auto": B.LLAMA_ATTN_AUTO, "chunked": B.LLAMA_ATTN_CHUNKED, "streamk": B.LLAMA_ATTN_STREAMK}
DECODE_ATTENTION = "auto"
CLOCK_LOG_DIR = os.environ.get("TMPDIR", "/tmp")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama7b-layer", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-log", default=None, help="directory for the per-rank clock sample CSV")
    ap.add_argument("--decode-kernel", default="auto", choices=sorted(DECODE_KERNELS),
                    help="decode-step launch structure (llama_set_decode_kernel)")
    ap.add_argument("--decode-attention", default="auto", choices=sorted(DECODE_ATTENTIONS),
                    help="decode attention kernel of the per-step launches (llama_set_decode_attention)")
    args = ap.parse_args()
    global DECODE_KERNEL, DECODE_ATTENTION, CLOCK_LOG_DIR
    DECODE_KERNEL = args.decode_kernel
    DECODE_ATTENTION = args.decode_attention
    if args.clock_log:
        CLOCK_LOG_DIR = args.clock_log
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup()
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
