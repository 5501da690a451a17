"""Host-side logic of bench.py on CPU: the multi-rank time reduction over a
2-rank gloo group, the whole-job aggregate, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]
        m = bench.max_over_ranks(ms, world, device="cpu")
        v = bench.job_throughput(640, 10, m, world)
        out.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 20.0                                  # the slower rank's time on every rank
        assert abs(v - 2 * 640 * 10 / 0.020) < 1e-6       # all ranks' tokens over that time


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny-fp32", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3


def test_decode_launch_count_per_block():
    """The `gpu_launches` claim: 5 kernels per block and decode step where the
    GEMVs compute the RMSNorms (bf16, at most 4 tokens, dim <= 4096), 7 where the
    RMSNorms are launches of their own, 1 for the persistent decode kernel."""
    import bench
    from llama_decoder_block_kv_b200 import synth
    w7 = synth.WORKLOADS["llama7b-layer"]
    w70 = synth.WORKLOADS["llama70b-layer"]
    w8 = synth.WORKLOADS["llama3-8b-decode"]
    wt = synth.WORKLOADS["tiny-fp32"]
    assert bench.decode_launches_per_block(w7, 1) == 5
    assert bench.decode_launches_per_block(w7, 4) == 5
    assert bench.decode_launches_per_block(w7, 5) == 7
    assert bench.decode_launches_per_block(w70, 16) == 7    # dim 8192
    assert bench.decode_launches_per_block(w8, 32) == 7     # 32 tokens
    assert bench.decode_launches_per_block(wt, 1) == 7      # fp32: the SIMT path
    saved = bench.DECODE_KERNEL
    try:
        bench.DECODE_KERNEL = "persistent"
        assert bench.decode_launches_per_block(w7, 1) == 1
        assert bench.decode_launches_per_block(wt, 1) == 7
    finally:
        bench.DECODE_KERNEL = saved
