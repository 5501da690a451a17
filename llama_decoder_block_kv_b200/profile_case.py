"""Run one kernel case repeatedly (for profilers and quick timing).

  python -m llama_decoder_block_kv_b200.profile_case gemv M N K [--reps R] [--graph]
  python -m llama_decoder_block_kv_b200.profile_case tc   M N K [--reps R]
  python -m llama_decoder_block_kv_b200.profile_case simt M N K [--reps R]
  python -m llama_decoder_block_kv_b200.profile_case prefill-attn T [--batch B] [--shape 7b|8b]
                                                     (LLaMA-7B or LLaMA-3-8B layer shape, one block call)
  python -m llama_decoder_block_kv_b200.profile_case decode-attn B L [--decode-attention chunked|streamk|auto]
                                                     (LLaMA-2-70B layer shape, one block call)

GEMM cases call llama_linear on seeded bf16 inputs; the block cases call
llama_block_forward. Prints the mean CUDA-event time per launch.
"""
from __future__ import annotations

import argparse

import torch

from . import binding as B
from . import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["gemv", "tc", "simt", "prefill-attn", "decode-attn"])
    ap.add_argument("sizes", type=int, nargs="+")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--graph", action="store_true", help="time the launches inside one CUDA graph")
    ap.add_argument("--decode-attention", default="auto", choices=["auto", "chunked", "streamk"],
                    help="decode-attn: the attention kernel of the call (llama_set_decode_attention)")
    ap.add_argument("--shape", default="7b", choices=["7b", "8b"],
                    help="prefill-attn: the LLaMA-7B layer (MHA) or the LLaMA-3-8B layer (GQA 32/8)")
    ap.add_argument("--batch", type=int, default=1, help="prefill-attn: sequences of T tokens")
    ap.add_argument("--gemv-mma", default="auto", choices=["auto", "warp", "tcgen05"],
                    help="gemv: the product of 9..32-token calls (llama_set_decode_linear_mma)")
    ap.add_argument("--row-major", action="store_true",
                    help="gemv / tc: pass the weights row-major instead of in the library's tile layout")
    a = ap.parse_args()
    torch.cuda.set_device(0)
    B.llama_set_decode_linear_mma({"auto": B.LLAMA_GEMV_MMA_AUTO, "warp": B.LLAMA_GEMV_MMA_WARP,
                                   "tcgen05": B.LLAMA_GEMV_MMA_TCGEN05}[a.gemv_mma])
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.kind in ("gemv", "tc", "simt"):
        M, N, K = a.sizes
        x = synth.normal((M, K), 1.0, 1, torch.bfloat16, "cuda")
        # enough weight copies that consecutive launches never find their weights in L2 (126 MB)
        n_w = max(1, -(-400 * 2 ** 20 // (N * K * 2)))
        ws = [synth.normal((N, K), 0.02, 2 + i, torch.bfloat16, "cuda") for i in range(n_w)]
        y = torch.empty((M, N), device="cuda")
        path = {"gemv": B.LLAMA_PATH_GEMV, "tc": B.LLAMA_PATH_TCGEN05, "simt": B.LLAMA_PATH_SIMT}[a.kind]
        if a.kind != "simt" and not a.row_major:
            ws = [B.llama_tile_weights(w) for w in ws]
            path |= B.LLAMA_WEIGHTS_TILED
        for w in ws:
            B.llama_linear(x, w, y, path, n=N)
        torch.cuda.synchronize()
        if a.graph:
            # a graph of `reps` back-to-back launches: no host overhead between them
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(a.reps):
                    B.llama_linear(x, ws[i % n_w], y, path, n=N)
            g.replay()
            torch.cuda.synchronize()
            e0.record(st)
            g.replay()
            e1.record(st)
        else:
            e0.record(st)
            for i in range(a.reps):
                B.llama_linear(x, ws[i % n_w], y, path, n=N)
            e1.record(st)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / a.reps
        flops = 2.0 * M * N * K
        byts = 2.0 * (M * K + N * K) + 4.0 * M * N
        print(f"{a.kind} M={M} N={N} K={K}: {ms * 1e3:.1f} us/launch, {flops / ms / 1e9:.1f} TFLOP/s, "
              f"{byts / ms / 1e6:.1f} GB/s")
        return
    if a.kind == "prefill-attn":
        T = a.sizes[0]
        if a.shape == "7b":
            w = synth.LLAMA7B_LAYER.with_(max_batch_size=a.batch, max_seq_len=max(T, 2048))
        else:
            w = synth.LLAMA3_8B_PREFILL.with_(n_layers=1, vocab_size=0, max_batch_size=a.batch,
                                              max_seq_len=max(T, 2048))
        m = B.Llama(B.ModelArgs.from_workload(w))
        B.llama_set_layer(m.ctx, 0, synth.layer_weights(w, 0, device="cuda"))
        h0 = synth.hidden(w, (a.batch, T, w.dim), 0, "cuda")
        pos = 0
    else:
        w = synth.LLAMA70B_LAYER
        Bsz, L = a.sizes
        m = B.Llama(B.ModelArgs.from_workload(w.with_(max_batch_size=Bsz)))
        B.llama_set_decode_attention(m.ctx, {"auto": B.LLAMA_ATTN_AUTO, "chunked": B.LLAMA_ATTN_CHUNKED,
                                             "streamk": B.LLAMA_ATTN_STREAMK}[a.decode_attention])
        B.llama_set_layer(m.ctx, 0, synth.layer_weights(w, 0, device="cuda"))
        h0 = synth.hidden(w, (Bsz, 1, w.dim), 0, "cuda")
        pos = L
    h = h0.clone()
    B.llama_block_forward(m.ctx, 0, h, pos)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(a.reps):
        h.copy_(h0)
        B.llama_block_forward(m.ctx, 0, h, pos)
    e1.record(st)
    e1.synchronize()
    print(f"{a.kind} {a.sizes}: {e0.elapsed_time(e1) / a.reps * 1e3:.1f} us per block call")
    code, flags = B.llama_get_error(m.ctx)
    m.close()
    if code != B.LLAMA_OK:
        raise SystemExit(f"device flag: {B.strerror(code)}")


if __name__ == "__main__":
    main()
