#!/usr/bin/env python
"""Benchmark of the LLaMA decoder-block library on B200.

Default workload (one step): a LLaMA-1-7B-shaped decoder layer in bf16
(dim 4096, 32 heads, MHA, ffn 11008), batch 1: a 512-token prefill from
start_pos 0, then 128 single-token decode steps at positions 512..639, all
through llama_block_forward. The 128 decode steps of a pass are captured in
one CUDA graph together with the prefill; the graph also restores the step's
inputs first, so every step does identical work. Prints one JSON line.

At one GPU the line also carries a "configs" object with the other
workloads (the tiny fp32 model, the LLaMA-2-70B-shaped layer decode, the
LLaMA-3-8B-shaped ragged decode and 4 x 8192 prefill), each with its
device-timed throughput, clocks, the roofline of its dominant kernel, an
end-to-end number with host buffers and the oracle's CPU baseline on a
stated sample (--configs none skips them).

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

def decode_launches_per_block(w, tokens: int) -> int:
    """Kernels of one block's decode step of `tokens` tokens: one persistent launch (bf16, when
    chosen); else gemv, attention (chunk merge fused), gemv, gemv, gemv and the two RMSNorms, which
    run inside the GEMVs that read them for bf16 calls of at most 4 tokens at dim <= 4096."""
    if w.act != "bf16":
        return 7
    if DECODE_KERNEL == "persistent":
        return 1
    return 5 if (tokens <= 4 and w.dim <= 4096 and w.dim % 64 == 0) else 7


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
        return pre + self.ND * decode_launches_per_block(self.w, self.Bsz)

    def decode_gemms(self):
        """(x, w) pairs of the decode linears, same shapes and kernel as the decode path."""
        return layer_pairs(self.w, self.Bsz)

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


def linear_roofline(pairs, path, peaks, reps, kernel, bound="hbm", peak_key="hbm_gbs", traffic_ratio=None,
                    traffic_source=None):
    """Average rate of one GEMM kernel of the library: the (x, w) pairs (a layer's
    linears, the weights in the tile layout the library keeps) launched back to
    back ``reps`` times inside one CUDA graph, timed with CUDA events around the
    replay on the launching stream. Algorithmic work per launch: for an HBM-bound
    kernel the weights + activations in + fp32 outputs, for a tensor-bound one
    2*M*N*K FLOP."""
    ys = [torch.empty((x.shape[0], w.shape[0]), device="cuda") for x, w in pairs]
    if bound == "hbm":
        work = sum(w.numel() * 2 + x.numel() * 2 + x.shape[0] * w.shape[0] * 4 for x, w in pairs)
    else:
        work = sum(2.0 * x.shape[0] * w.shape[0] * x.shape[1] for x, w in pairs)
    tiles = [(x, B.llama_tile_weights(w), w.shape[0]) for x, w in pairs]
    path = path | B.LLAMA_WEIGHTS_TILED
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
    per_launch = work / len(pairs)
    if bound == "hbm":
        achieved, unit = per_launch / (t_ms * 1e-3) / 1e9, "GB/s"
    else:
        achieved, unit = per_launch / (t_ms * 1e-3) / 1e12, "TFLOP/s"
    peak = peaks[peak_key]
    out = {"kernel": kernel, "bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4),
           "traffic": None if traffic_ratio is None else int(round(traffic_ratio * per_launch)),
           ("bytes_per_launch" if bound == "hbm" else "flop_per_launch"): int(per_launch),
           "avg_launch_us": round(t_ms * 1e3, 2), "launches_timed": launches, "peak_key": peak_key}
    if traffic_source:
        out["traffic_source"] = traffic_source
    del g
    return out


def gemv_roofline(lb: "LayerBench", peaks, reps=10):
    """The decode GEMV over the layer's four decode linears (wqkv, wo, w1|w3, w2),
    larger than L2 together (405 MB for the LLaMA-7B layer)."""
    return linear_roofline(lb.decode_gemms(), B.LLAMA_PATH_GEMV, peaks, reps,
                           "llama_decode_linear_kernel (decode linears: wqkv, wo, w1|w3, w2)",
                           traffic_ratio=GEMV_TRAFFIC_RATIO,
                           traffic_source="ncu dram read+write of the w1|w3 launch scaled by algorithmic bytes "
                                          "(M=1, N=22016, K=4096)")


def layer_pairs(w: synth.Workload, M: int, layer: int = 0):
    """(x, w) pairs of one block's linears as the library packs them: wq|wk|wv,
    wo, w1|w3 row-interleaved, w2; x seeded N(0, 1) bf16 with M rows."""
    lw = synth.layer_weights(w, layer, device="cuda")
    wqkv = torch.cat([lw["wq"], lw["wk"], lw["wv"]], 0).contiguous()
    w13 = torch.stack([lw["w1"], lw["w3"]], 1).reshape(2 * w.ffn_hidden, w.dim).contiguous()
    xs = {K: synth.normal((M, K), 1.0, 7 + K, torch.bfloat16, "cuda")
          for K in (w.dim, w.ffn_hidden, w.n_heads * w.head_dim)}
    return [(xs[w.dim], wqkv), (xs[w.n_heads * w.head_dim], lw["wo"]), (xs[w.dim], w13),
            (xs[w.ffn_hidden], lw["w2"])]


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


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _bits(t):
    """bf16 tensor -> raw uint16 patterns (the oracle widens them slice by slice)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_model(w: synth.Workload, n_layers: int, **over):
    import oracle as O
    a = O.ModelArgs(dim=w.dim, n_layers=n_layers, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                    vocab_size=w.vocab_size, multiple_of=w.multiple_of, ffn_dim_multiplier=w.ffn_dim_multiplier,
                    norm_eps=w.norm_eps, rope_theta=w.rope_theta, max_batch_size=w.max_batch_size,
                    max_seq_len=w.max_seq_len, act=w.act)
    for k, v in over.items():
        setattr(a, k, v)
    m = O.OracleModel(a)
    for i in range(n_layers):
        m.layers[i] = {k: _f64(v) for k, v in synth.layer_weights(w, i, device="cuda").items()}
    if w.vocab_size:
        enh = synth.embed_norm_head(w, device="cuda")
        m.tok_embeddings, m.norm, m.output = _bits(enh["tok_embeddings"]), _f64(enh["norm"]), _bits(enh["output"])
        if w.act == "fp32":
            m.tok_embeddings, m.output = _f64(enh["tok_embeddings"]), _f64(enh["output"])
    return m


def oracle_sample(name: str, w: synth.Workload):
    """The oracle (numpy float64, as it stands) timed on the host cores on a bounded
    sample of a workload; returns the cpu_baseline object (tokens/s)."""
    import oracle as O
    threads = _oracle_threads()
    if name == "tiny-fp32":
        m = _oracle_model(w, w.n_layers)
        tok = _f64(synth.tokens(w, (w.batch, w.prefill_len + w.decode_steps), 0, "cuda")).astype(np.int64)
        t0 = time.perf_counter()
        m.forward(tok[:, :w.prefill_len], 0)
        for s in range(w.decode_steps):
            p = w.prefill_len + s
            m.forward(tok[:, p:p + 1], p)
        t = time.perf_counter() - t0
        return {"value": round(w.batch * (w.prefill_len + w.decode_steps) / t, 2), "unit": "tokens/s",
                "cores": threads, "kind": "oracle", "sample": "the whole run: prefill of 32 tokens and 16 decode steps"}
    if name == "llama70b-layer":
        t, threads, sample = oracle_layer_sample(w, n_decode=1)
        return {"value": round(w.batch * w.decode_steps / t, 2), "unit": "tokens/s", "cores": threads,
                "kind": "oracle", "sample": "one decode step of batch 16 over the 4096-position cache (the full step)"}
    if name == "llama3-8b-decode":
        L = 2
        m = _oracle_model(w, L)
        lens = _f64(synth.ragged_lengths(w, "cuda")).astype(np.int64)
        shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
        for i in range(L):
            m.cache_k[i][...] = _f64(synth.cache_values(w, i, 0, shape, "cuda"))
            m.cache_v[i][...] = _f64(synth.cache_values(w, i, 1, shape, "cuda"))
        tok = _f64(synth.tokens(w, (w.decode_steps, w.batch), 0, "cuda")).astype(np.int64)[0]
        t0 = time.perf_counter()
        h = O.as_f64(m.tok_embeddings[tok]).reshape(w.batch, 1, w.dim)
        t_embed = time.perf_counter() - t0
        t_layers = []
        for i in range(L):
            t0 = time.perf_counter()
            h = m.block(i, h, lens)
            t_layers.append(time.perf_counter() - t0)
        t0 = time.perf_counter()
        m._lm_head(O.rmsnorm(h, m.norm, w.norm_eps, w.act))
        t_head = time.perf_counter() - t0
        t_step = t_embed + w.n_layers * (sum(t_layers) / L) + t_head
        return {"value": round(w.batch / t_step, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": "one decode step of the 32 sequences (ragged, first of the 64 steps) over 2 of the 32 "
                          "layers + the final norm and LM head, timed; the per-layer time scaled to 32 layers"}
    if name == "llama3-8b-prefill":
        L, T = 2, 1024
        m = _oracle_model(w, L, max_batch_size=1, max_seq_len=T)
        tok = _f64(synth.tokens(w, (w.batch, w.prefill_len), 0, "cuda")).astype(np.int64)[:1, :T]
        t0 = time.perf_counter()
        m.forward(tok, 0, all_positions=False)
        t = time.perf_counter() - t0
        return {"value": round(T / t, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": "a reduced prefill: 1 x 1024 tokens through 2 layers of the same dims + the final norm "
                          "and last-position LM head (the full 4 x 8192 x 32-layer prefill is ~528 TFLOP)"}
    raise ValueError(name)


CONFIG_STEPS = {"tiny-fp32": (20, 3), "llama70b-layer": (50, 3), "llama3-8b-decode": (3, 3),
                "llama3-8b-prefill": (3, 3)}


def run_configs(args, world, local, peaks, peak_kind, names):
    """The other workloads, one object each: device-timed value, clocks, the
    dominant kernel's roofline, end to end with host buffers, and the oracle's
    CPU baseline (rank 0 at one GPU)."""
    out = {}
    for name in names:
        w = synth.WORKLOADS[name]
        steps, warmup = CONFIG_STEPS[name]
        if w.n_layers == 1:
            lb = LayerBench(w)
            g = lb.capture("all")
            sampler = NvmlClockSampler(local)
            barrier(world)
            sampler.start()
            ms = max_over_ranks(time_graph(g, steps, warmup, world), world)
            clocks = sampler.stop()
            ms_step = ms / steps
            wbytes = 2 * (w.dim * (w.n_heads + 2 * w.n_kv_heads) * w.head_dim + w.n_heads * w.head_dim * w.dim +
                          3 * w.dim * w.ffn_hidden)
            kv = w.batch * (w.cache_len + 1) * 2 * w.n_kv_heads * w.head_dim * 2
            r = {"workload": w.name, "value": round(world * lb.tokens_per_step * steps / (ms * 1e-3), 1),
                 "unit": "tokens/s", "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4),
                 "clocks": clocks, "gpu_launches": lb.kernels_per_step() * steps,
                 "phases": {"weights_gb": round(wbytes / 1e9, 3), "kv_gb": round(kv / 1e9, 4),
                            "hbm_gbs": round((wbytes + kv) / (ms_step * 1e-3) / 1e9, 1),
                            "hbm_frac": round((wbytes + kv) / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}}
            r["roofline"] = linear_roofline(lb.decode_gemms(), B.LLAMA_PATH_GEMV, peaks, 5,
                                            "llama_decode_linear_kernel (the 70B layer's decode linears at 16 "
                                            "tokens: wqkv, wo, w1|w3, w2)")
            r["roofline"]["peak_kind"] = peak_kind
            r["e2e"] = run_e2e(lb, g, argparse.Namespace(steps=steps, warmup=warmup), world)
            del g
            lb.close()
        else:
            mb = ModelBench(w)
            r = model_config_entry(mb, steps, warmup, world, local, peaks, peak_kind)
            r["e2e"] = run_e2e_graph(mb.graph, mb.inputs, mb.outputs(), mb.tokens_per_step,
                                     argparse.Namespace(steps=steps, warmup=warmup), world)
            mb.close()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        if world == 1 and not args.no_cpu_baseline:
            r["cpu_baseline"] = oracle_sample(name, w)
        out[name] = r
    return out


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
           "data": "synthetic: seeded N(0,1) hidden states, N(0,0.02) weights, RMSNorm weights 1 (as the workloads state)",
           "config": {"workload": w.name, "batch": lb.Bsz, "prefill_tokens": lb.P, "decode_steps": lb.ND,
                      "decode_start_pos": lb.dec_pos0, "l2": "inputs larger than L2: %.0f MB of weights per pass"
                      % (wbytes / 1e6), "parallelism": "replicas" if world > 1 else "single GPU",
                      "decode_kernel": DECODE_KERNEL, "decode_attention": DECODE_ATTENTION},
           "phases": phases, "roofline": roof, "e2e": e2e,
           "gpu_launches": lb.kernels_per_step() * args.steps, "clocks": clocks}
    del g
    lb.close()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, threads, sample = oracle_layer_sample(w)
        out["cpu_baseline"] = {"value": round(lb.tokens_per_step / t_cpu, 2), "unit": "tokens/s", "cores": threads,
                               "kind": "oracle", "sample": sample}
    if world == 1 and args.configs != "none":
        names = [n for n in ("tiny-fp32", "llama70b-layer", "llama3-8b-decode", "llama3-8b-prefill")
                 if n != args.workload and (args.configs == "all" or n in args.configs.split(","))]
        out["configs"] = run_configs(args, world, local, peaks, peak_kind, names)
    return out


def run_e2e(lb: LayerBench, g, args, world):
    """Same metric with host buffers: pinned H2D of inputs and D2H of outputs inside the timed region."""
    ins = [t for t in (lb.h_pre0, lb.h_dec0) if t is not None]
    outs = [t for t in (lb.h_pre, lb.h_dec) if t is not None]
    return run_e2e_graph(g, ins, outs, lb.tokens_per_step, args, world)


class ModelBench:
    """A whole model (embedding, blocks, final norm, LM head) through llama_forward /
    llama_forward_ragged, one step captured in a CUDA graph:
      - the tiny fp32 model: a 32-token prefill then 16 decode steps, all-position logits;
      - the LLaMA-3-8B shape, ragged decode: 64 decode steps of a batch of 32 at
        per-sequence positions (caches prefilled with N(0,1) to uniform lengths);
      - the LLaMA-3-8B shape, prefill: 4 x 8192 tokens from start_pos 0, last-position logits."""

    def __init__(self, w: synth.Workload):
        self.w = w
        self.m = B.Llama(B.ModelArgs.from_workload(w))
        ctx = self.ctx = self.m.ctx
        B.llama_set_decode_kernel(ctx, DECODE_KERNELS[DECODE_KERNEL])
        B.llama_set_decode_attention(ctx, DECODE_ATTENTIONS[DECODE_ATTENTION])
        for i in range(w.n_layers):
            B.llama_set_layer(ctx, i, synth.layer_weights(w, i, device="cuda"))
        enh = synth.embed_norm_head(w, device="cuda")
        B.llama_set_embed_norm_head(ctx, enh["tok_embeddings"], enh["norm"], enh["output"])
        del enh
        per_block = decode_launches_per_block(w, w.batch)
        if w.ragged_hi:                      # ragged decode from prefilled caches
            self.kind = "ragged-decode"
            self.lens = synth.ragged_lengths(w, "cuda")
            shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
            for i in range(w.n_layers):
                k = synth.cache_values(w, i, 0, shape, "cuda")
                v = synth.cache_values(w, i, 1, shape, "cuda")
                B.llama_kv_write(ctx, i, k, v)
                del k, v
            self.toks = synth.tokens(w, (w.decode_steps, w.batch), 0, "cuda")
            steps = torch.arange(w.decode_steps, device="cuda", dtype=torch.int32)[:, None]
            self.pos = (self.lens[None, :] + steps).contiguous()
            self.logits = torch.empty((w.batch, w.vocab_size), device="cuda")
            B.llama_reserve(ctx, w.batch)
            self.tokens_per_step = w.batch * w.decode_steps
            self.launches_per_step = w.decode_steps * (1 + w.n_layers * per_block + 2)
            self.inputs = [self.toks, self.pos]
        elif w.decode_steps:                 # prefill then decode steps, all-position logits
            self.kind = "prefill+decode"
            P, ND = w.prefill_len, w.decode_steps
            self.toks = synth.tokens(w, (w.batch, P + ND), 0, "cuda")
            self.logits_pre = torch.empty((w.batch, P, w.vocab_size), device="cuda")
            self.logits_dec = torch.empty((ND, w.batch, 1, w.vocab_size), device="cuda")
            if w.batch != 1:
                raise ValueError("the prefill+decode model step reads its decode tokens as views (batch 1)")
            B.llama_reserve(ctx, w.batch * P)
            self.tokens_per_step = w.batch * (P + ND)
            blocks = 1 + w.n_layers * 7 + 2
            self.launches_per_step = blocks + ND * (1 + w.n_layers * per_block + 2)
            self.inputs = [self.toks]
        else:                                # one long prefill, last-position logits
            self.kind = "prefill"
            self.toks = synth.tokens(w, (w.batch, w.prefill_len), 0, "cuda")
            self.logits = torch.empty((w.batch, w.vocab_size), device="cuda")
            B.llama_reserve(ctx, w.batch * w.prefill_len)
            self.tokens_per_step = w.batch * w.prefill_len
            self.launches_per_step = 1 + w.n_layers * 7 + 2
            self.inputs = [self.toks]
        self.enqueue()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.enqueue()
        torch.cuda.synchronize()

    def enqueue(self):
        w, ctx = self.w, self.ctx
        if self.kind == "ragged-decode":
            for s in range(w.decode_steps):
                B.llama_forward_ragged(ctx, self.toks[s], self.pos[s], self.logits)
        elif self.kind == "prefill+decode":
            P = w.prefill_len
            B.llama_forward(ctx, self.toks[:, :P], 0, self.logits_pre, True)
            for s in range(w.decode_steps):
                B.llama_forward(ctx, self.toks[:, P + s:P + s + 1], P + s, self.logits_dec[s], True)
        else:
            B.llama_forward(ctx, self.toks, 0, self.logits, False)

    def outputs(self):
        if self.kind == "prefill+decode":
            return [self.logits_pre, self.logits_dec]
        return [self.logits]

    def close(self):
        del self.graph
        self.m.close()


def run_e2e_graph(g, inputs, outputs, tokens_per_step, args, world, steps=None):
    """The step through the C ABI with host buffers: every step's inputs are
    copied from pinned host memory to the device and its results back to
    pinned host memory, all inside the timed region (`h2d_bytes_per_step`,
    `d2h_bytes_per_step`).

    `value`: the copies run on a second stream, overlapped with the
    neighbouring steps' compute, as a serving loop would: step t + 1's inputs
    go up into one of two device staging slots while step t computes, and step
    t's results come down from a staging slot while step t + 1 computes. On the
    compute stream each step copies its staged inputs into the graph's input
    buffers, replays the graph and copies the results into the staging slot
    (two device-to-device copies of the step's inputs and outputs). The region
    ends when the last step's results are in host memory.
    `serial_value`: the same copies in line on the compute stream, no overlap."""
    steps = args.steps if steps is None else steps
    hin = [t.cpu().pin_memory() for t in inputs]
    hout = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outputs] for _ in range(2)]
    stage_in = [[torch.empty_like(t) for t in inputs] for _ in range(2)]
    stage_out = [[torch.empty_like(t) for t in outputs] for _ in range(2)]
    st = torch.cuda.current_stream()
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]       # a slot's inputs landed
    ev_in_free = [torch.cuda.Event() for _ in range(2)]  # a slot's inputs copied into the graph's buffers
    ev_out = [torch.cuda.Event() for _ in range(2)]      # a slot's results staged
    ev_d2h = [torch.cuda.Event() for _ in range(2)]      # a slot's results in host memory

    def h2d(t):
        s = t % 2
        with torch.cuda.stream(cs):
            if t >= 2:
                cs.wait_event(ev_in_free[s])
            for d, h in zip(stage_in[s], hin):
                d.copy_(h, non_blocking=True)
            ev_in[s].record(cs)

    def compute(t):
        s = t % 2
        st.wait_event(ev_in[s])
        for d, src in zip(inputs, stage_in[s]):
            d.copy_(src)
        ev_in_free[s].record(st)
        g.replay()
        if t >= 2:
            st.wait_event(ev_d2h[s])
        for d, src in zip(stage_out[s], outputs):
            d.copy_(src)
        ev_out[s].record(st)

    def d2h(t):
        s = t % 2
        with torch.cuda.stream(cs):
            cs.wait_event(ev_out[s])
            for h, src in zip(hout[s], stage_out[s]):
                h.copy_(src, non_blocking=True)
            ev_d2h[s].record(cs)

    def pipelined(n):
        cs.wait_stream(st)
        h2d(0)
        for t in range(n):
            if t + 1 < n:
                h2d(t + 1)
            compute(t)
            d2h(t)
        st.wait_stream(cs)

    def serial(n):
        for _ in range(n):
            for d, h in zip(inputs, hin):
                d.copy_(h, non_blocking=True)
            g.replay()
            for h, d in zip(hout[0], outputs):
                h.copy_(d, non_blocking=True)

    def timed(run, n):
        run(args.warmup)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        run(n)
        e1.record(st)
        e1.synchronize()
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world)

    ms = timed(pipelined, steps)
    ms_serial = timed(serial, steps)
    tok = world * tokens_per_step * steps
    return {"value": round(tok / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in inputs)),
            "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outputs)),
            "copies": "overlapped with the neighbouring steps on a second stream",
            "serial_value": round(tok / (ms_serial * 1e-3), 1)}


def run_model_bench(args, world, rank, local, w, peaks, peak_kind):
    """A whole-model workload as the headline line (--workload llama3-8b-*)."""
    mb = ModelBench(w)
    r = model_config_entry(mb, args.steps, args.warmup, world, local, peaks, peak_kind)
    out = {"metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f32" if w.act == "fp32" else "bf16", "data": "synthetic",
           "config": {"workload": w.name, "decode_kernel": DECODE_KERNEL, "decode_attention": DECODE_ATTENTION},
           "phases": r.get("phases", {}), "roofline": r["roofline"], "clocks": r["clocks"],
           "gpu_launches": r["gpu_launches"]}
    out["e2e"] = run_e2e_graph(mb.graph, mb.inputs, mb.outputs(), mb.tokens_per_step, args, world)
    mb.close()
    return out


def model_config_entry(mb: ModelBench, steps, warmup, world, local, peaks, peak_kind):
    """Time a whole-model step and measure its dominant kernel."""
    w = mb.w
    sampler = NvmlClockSampler(local)
    barrier(world)
    sampler.start()
    ms = max_over_ranks(time_graph(mb.graph, steps, warmup, world), world)
    clocks = sampler.stop()
    code, flags = B.llama_get_error(mb.ctx)
    if code != B.LLAMA_OK:
        raise RuntimeError(f"device flag raised during the timed steps: {B.strerror(code)} ({flags})")
    ms_step = ms / steps
    r = {"workload": w.name, "value": round(world * mb.tokens_per_step * steps / (ms * 1e-3), 1),
         "unit": "tokens/s", "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4),
         "clocks": clocks, "gpu_launches": mb.launches_per_step * steps}
    D, H, Hkv, F = w.head_dim, w.n_heads, w.n_kv_heads, w.ffn_hidden
    layer_params = w.dim * (H + 2 * Hkv) * D + H * D * w.dim + 3 * w.dim * F
    if mb.kind == "ragged-decode":
        wbytes = 2 * (w.n_layers * layer_params + w.vocab_size * w.dim)
        lens = mb.lens.double()
        kv = sum(float((lens + s + 1).sum()) for s in range(w.decode_steps)) * w.n_layers * 2 * Hkv * D * 2
        byts = w.decode_steps * wbytes + kv
        r["phases"] = {"weights_gb_per_decode_step": round(wbytes / 1e9, 3),
                       "kv_gb_per_decode_step": round(kv / w.decode_steps / 1e9, 3),
                       "hbm_gbs": round(byts / (ms_step * 1e-3) / 1e9, 1),
                       "hbm_frac": round(byts / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
        r["roofline"] = linear_roofline(layer_pairs(w, w.batch), B.LLAMA_PATH_GEMV, peaks, 5,
                                        "llama_decode_linear_kernel (the 8B layer's decode linears at 32 tokens)")
    elif mb.kind == "prefill":
        T = w.prefill_len
        flops = 2.0 * w.batch * T * w.n_layers * layer_params
        flops += w.n_layers * w.batch * 4.0 * H * D * (T * (T + 1) / 2)
        flops += 2.0 * w.batch * w.dim * w.vocab_size
        r["phases"] = {"tflops": round(flops / (ms_step * 1e-3) / 1e12, 1),
                       "tensor_frac_sustained": round(flops / (ms_step * 1e-3) / 1e12
                                                      / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4)}
        r["roofline"] = linear_roofline(layer_pairs(w, w.batch * T), B.LLAMA_PATH_TCGEN05, peaks, 2,
                                        "gemm_tc_kernel (the 8B layer's prefill linears at 32768 tokens)",
                                        bound="tensor", peak_key="bf16_tflops_sustained"
                                        if "bf16_tflops_sustained" in peaks else "bf16_tflops")
    else:   # the tiny fp32 model: latency-bound, 2.08 M parameters
        n_fwd = 1 + w.decode_steps
        wbytes = 4 * (w.n_layers * layer_params + 2 * w.vocab_size * w.dim)
        achieved = n_fwd * wbytes / (ms_step * 1e-3) / 1e9
        r["roofline"] = {"kernel": "whole step (latency-bound: %d launches of a 2-layer dim-256 model)"
                         % mb.launches_per_step, "bound": "hbm", "achieved": round(achieved, 2),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 5),
                         "traffic": None, "bytes_per_step": n_fwd * wbytes}
    r["roofline"]["peak_kind"] = peak_kind
    return r


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
    ap.add_argument("--configs", default="all",
                    help="the other workloads reported under 'configs' at one GPU: all, none, or a comma list")
    ap.add_argument("--clock-log", default=None, help="directory for the per-rank clock sample CSV")
    ap.add_argument("--decode-kernel", default="auto", choices=sorted(DECODE_KERNELS),
                    help="decode-step launch structure (llama_set_decode_kernel)")
    ap.add_argument("--gemv-mma", default="auto", choices=["auto", "warp", "tcgen05"],
                    help="product of the 9..32-token decode GEMV (llama_set_decode_linear_mma)")
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
    B.llama_set_decode_linear_mma({"auto": B.LLAMA_GEMV_MMA_AUTO, "warp": B.LLAMA_GEMV_MMA_WARP,
                                   "tcgen05": B.LLAMA_GEMV_MMA_TCGEN05}[args.gemv_mma])
    world, rank, local = dist_setup()
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
