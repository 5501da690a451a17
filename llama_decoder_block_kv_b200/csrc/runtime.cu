// Host runtime and C ABI (include/llama_b200.h): owns the packed weights, the
// KV-caches, the RoPE table and the workspace, validates every call, and
// enqueues the kernels of one forward pass on the caller's stream.
//
// Per block ("LLaMA: Open and Efficient Foundation Language Models" notes,
// TransformerBlock.forward):
//   rmsnorm(h) -> xn
//   xn * Wqkv^T  -> RoPE(q) -> q buffer; RoPE(k), v -> cache slots       (QKV epilogue)
//   attention(q, cache) -> o                                             (prefill or split-K decode)
//   h += o * Wo^T                                                        (residual epilogue)
//   rmsnorm(h) -> xn
//   xn * W13^T -> silu(a) * b -> g                                       (SwiGLU epilogue)
//   h += g * W2^T                                                        (residual epilogue)
// Whole-model calls add the embedding gather before and the final RMSNorm
// plus the LM head after ("... notes", Transformer.forward). A decode call of
// at most 4 tokens at dim <= 4096 computes each rmsnorm inside the GEMV that
// reads xn (same arithmetic, no launch of its own).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "kernels.cuh"

using namespace llama;

namespace {

struct Layer {
  void* wqkv = nullptr;
  void* wo = nullptr;
  void* w13 = nullptr;
  void* w2 = nullptr;
  void* attn_norm = nullptr;
  void* ffn_norm = nullptr;
  void* cache_k = nullptr;
  void* cache_v = nullptr;
  CUtensorMap map_k, map_v;
  CUtensorMap map_w[4];  // wqkv, wo, w13, w2 as 128-row x 64-k TMA tiles (persistent decode kernel)
  bool set = false;
};

}  // namespace

struct llama_ctx {
  llama_args a;
  bool bf16 = true;
  bool half_split = false;  // weights given with half-split RoPE pairs
  int esz = 2;
  int dim = 0, H = 0, Hkv = 0, D = 0, n_rep = 1, F = 0, V = 0, S = 0, Bm = 0, L = 0;
  int n_qkv = 0;
  int device = 0, num_sms = 148;
  std::vector<Layer> layers;
  void* tok_emb = nullptr;
  void* final_norm = nullptr;
  void* output = nullptr;
  CUtensorMap map_out;  // the LM head as 128-row x 64-k TMA tiles (bf16)
  bool head_set = false;
  float2* rope = nullptr;
  int* err = nullptr;
  // workspace, sized for ws_tokens tokens
  int ws_tokens = 0;
  float* h = nullptr;
  void* xn = nullptr;
  void* q = nullptr;
  void* o = nullptr;
  void* g = nullptr;
  // scratch for split-K partial sums (GEMV) and decode-attention partials
  float* part = nullptr;
  size_t part_floats = 0;
  int* counters = nullptr;
  int counters_n = 0;
  GemmSplitWs split;  // the CTA-pair GEMM's two-way k split (prefill calls of few tiles), sized by reserve
  // persistent decode kernel: grid-barrier words and per-128-column sums of squares of h
  unsigned* gbar = nullptr;
  float* ssq = nullptr;
  int decode_mode = LLAMA_DECODE_AUTO;
  int attn_mode = LLAMA_ATTN_AUTO;
  // generation: last-position logits and sampling scratch, [max_batch][vocab] each;
  // the captured decode step's column counter and positions; its executable graph
  float* gen_logits = nullptr;
  float* gen_probs = nullptr;
  int* gen_state = nullptr;  // [0] column being generated, [1 .. max_batch] positions
  cudaGraphExec_t gen_exec = nullptr;
  cudaStream_t gen_exec_stream = nullptr;
};

namespace {

#define CK(call)                             \
  do {                                       \
    cudaError_t e_ = (call);                 \
    if (e_ != cudaSuccess) return LLAMA_ERR_CUDA; \
  } while (0)

// Every device allocation of the library goes through alloc / release, which
// keep the live total and honour the optional cap of llama_set_alloc_limit.
std::mutex g_alloc_mu;
std::unordered_map<void*, size_t> g_alloc_sizes;
uint64_t g_alloc_total = 0, g_alloc_limit = 0;

int alloc(void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return LLAMA_OK;
  std::lock_guard<std::mutex> lock(g_alloc_mu);
  if (g_alloc_limit && g_alloc_total + bytes > g_alloc_limit) return LLAMA_ERR_OOM;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    *p = nullptr;
    return LLAMA_ERR_OOM;
  }
  if (e != cudaSuccess) {
    *p = nullptr;
    return LLAMA_ERR_CUDA;
  }
  g_alloc_sizes[*p] = bytes;
  g_alloc_total += bytes;
  return LLAMA_OK;
}

void release(void*& p) {
  if (p) {
    cudaFree(p);
    std::lock_guard<std::mutex> lock(g_alloc_mu);
    auto it = g_alloc_sizes.find(p);
    if (it != g_alloc_sizes.end()) {
      g_alloc_total -= it->second;
      g_alloc_sizes.erase(it);
    }
  }
  p = nullptr;
}

int ffn_hidden(const llama_args* a) {
  if (a->dim <= 0 || a->multiple_of <= 0) return LLAMA_ERR_INVALID_ARGS;
  long hidden = 4L * a->dim;
  hidden = (long)(2.0 * (double)hidden / 3.0);
  if (a->ffn_dim_multiplier > 0.f) hidden = (long)((double)a->ffn_dim_multiplier * (double)hidden);
  const long mo = a->multiple_of;
  hidden = mo * ((hidden + mo - 1) / mo);
  if (hidden <= 0 || hidden > (1L << 30)) return LLAMA_ERR_INVALID_ARGS;
  return (int)hidden;
}

// RoPE angles as the pages' precompute_freqs_cis: freq_i = 1 / theta^(2i/D)
// (evaluated in double, rounded to fp32), angle = fp32(t) * freq_i (one fp32
// multiply, like torch.outer on fp32 vectors), cos/sin evaluated in double
// on that fp32 angle and rounded to fp32. Stored as (cos, sin) pairs.
std::vector<float2> rope_table(int D, int end, double theta) {
  std::vector<float2> t((size_t)end * (D / 2));
  std::vector<float> freq(D / 2);
  for (int i = 0; i < D / 2; ++i) freq[i] = (float)(1.0 / std::pow(theta, (double)(2 * i) / (double)D));
  for (int p = 0; p < end; ++p)
    for (int i = 0; i < D / 2; ++i) {
      volatile float ang = (float)p * freq[i];
      t[(size_t)p * (D / 2) + i] = make_float2((float)std::cos((double)ang), (float)std::sin((double)ang));
    }
  return t;
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// grid barrier of the persistent decode kernel: arrival counter and release word, 128 B apart
constexpr size_t kGbarBytes = 256;

int reserve(llama_ctx* c, int tokens) {
  if (tokens <= c->ws_tokens) return LLAMA_OK;
  cudaDeviceSynchronize();
  release(reinterpret_cast<void*&>(c->h));
  release(c->xn);
  release(c->q);
  release(c->o);
  release(c->g);
  c->ws_tokens = 0;
  const size_t T = (size_t)tokens;
  int r;
  if ((r = alloc(reinterpret_cast<void**>(&c->h), round256(T * c->dim * 4)))) return r;
  if ((r = alloc(&c->xn, round256(T * c->dim * c->esz)))) return r;
  if ((r = alloc(&c->q, round256(T * c->H * c->D * c->esz)))) return r;
  if ((r = alloc(&c->o, round256(T * c->H * c->D * c->esz)))) return r;
  if ((r = alloc(&c->g, round256(T * c->F * c->esz)))) return r;
  if (c->bf16 && tokens > 32) {  // calls of up to 32 tokens run the GEMV, not the GEMM
    // the split serves calls of at most gemm_split_max_tiles pair tiles: size it
    // for the most tiles one of the model's linears has at this many tokens
    const int Ns[5] = {c->n_qkv, c->dim, 2 * c->F, c->dim, c->V};
    int tiles = 0;
    for (int i = 0; i < 5; ++i)
      if (Ns[i] > 0) tiles = std::max(tiles, (int)((T + 255) / 256) * ((Ns[i] + 255) / 256));
    tiles = std::min(tiles, gemm_split_max_tiles(c->num_sms));
    if (tiles > c->split.tiles) {
      release(reinterpret_cast<void*&>(c->split.ws));
      release(reinterpret_cast<void*&>(c->split.sync));
      c->split.tiles = 0;
      if ((r = alloc(reinterpret_cast<void**>(&c->split.ws), gemm_split_ws_floats(tiles) * sizeof(float)))) return r;
      if ((r = alloc(reinterpret_cast<void**>(&c->split.sync), gemm_split_sync_ints(tiles) * sizeof(int)))) return r;
      if (cudaMemset(c->split.sync, 0, gemm_split_sync_ints(tiles) * sizeof(int)) != cudaSuccess)
        return LLAMA_ERR_CUDA;
      c->split.tiles = tiles;
    }
  }
  c->ws_tokens = tokens;
  return LLAMA_OK;
}

cudaStream_t S_(void* s) { return reinterpret_cast<cudaStream_t>(s); }

EpiParams epi_base(llama_ctx* c, int kind, int M, int N) {
  EpiParams p;
  std::memset(&p, 0, sizeof(p));
  p.kind = kind;
  p.M = M;
  p.N = N;
  p.err = c->err;
  return p;
}

// C[M][N] = A[M][K] * W[N][K]^T through the path that suits the shape.
// W is one of the library's weight matrices: row-major fp32 in fp32 mode,
// 128 x 64 bf16 tiles (tile_weights) in bf16 mode.
// wmap: W's tensor map (tiled layout, 128-row boxes), encoded when the weights were set.
// h_norm / w_norm (decode GEMV only, fuse_norm): A = RMSNorm(h_norm) computed by the GEMV itself.
bool gemm_is_gemv(const llama_ctx* c, int M, int K) { return c->bf16 && M <= 32 && K % 64 == 0; }
int gemm(llama_ctx* c, const void* A, const void* W, const CUtensorMap* wmap, int M, int N, int K, const EpiParams& ep,
         cudaStream_t st, const float* h_norm = nullptr, const void* w_norm = nullptr) {
  if (h_norm && !gemm_is_gemv(c, M, K)) return LLAMA_ERR_INVALID_ARGS;
  if (!c->bf16) {
    launch_gemm_simt<float>(A, W, M, N, K, ep, st);
    return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
  }
  if (gemm_is_gemv(c, M, K)) {
    GemvPlan p = plan_gemv(M, N, K, c->num_sms);
    if (p.part_floats > c->part_floats || p.row_blocks > c->counters_n) return LLAMA_ERR_INVALID_ARGS;
    return launch_gemv_bf16(A, W, 1, M, N, K, p, c->part, c->counters, ep, c->num_sms, st, wmap, h_norm, w_norm,
                            c->a.norm_eps) == cudaSuccess
               ? LLAMA_OK
               : LLAMA_ERR_CUDA;
  }
  return launch_gemm_tc(A, W, 1, M, N, K, ep, c->num_sms, st, wmap, &c->split) == cudaSuccess ? LLAMA_OK
                                                                                             : LLAMA_ERR_CUDA;
}

// A decode call of a few tokens (bf16, dim <= 4096) computes both RMSNorms
// inside the GEMVs that read them: no RMSNorm launch, no xn round trip.
bool fuse_norm(const llama_ctx* c, int M) { return gemm_is_gemv(c, M, c->dim) && gemv_can_fuse_norm(M, c->dim); }

// elements of one stored weight matrix [N][K]: tiles in bf16 mode, row-major in fp32 mode
size_t weight_elems(const llama_ctx* c, size_t N, size_t K) { return c->bf16 ? tiled_weight_elems(N, K) : N * K; }

// One decode step of a block in one persistent launch (decode_block.cu), when
// the call and the shapes allow it. Returns 1 when the call must take the
// kernel-per-step path instead.
int run_block_persistent(llama_ctx* c, int layer, float* h, int B, const int* sp_dev, int sp_host,
                         cudaStream_t st) {
  const int max_len = sp_dev ? c->S : sp_host + 1;
  DecodeBlockPlan pl = plan_decode_block(B, c->dim, c->H, c->Hkv, c->D, c->F, c->S, max_len, c->num_sms);
  if (!pl.ok || pl.part_floats > c->part_floats || pl.counters > c->counters_n) return 1;
  Layer& Ly = c->layers[layer];
  DecodeBlockParams p;
  std::memset(&p, 0, sizeof(p));
  for (int i = 0; i < 4; ++i) p.lin[i] = pl.lin[i];
  p.M = B;
  p.dim = c->dim;
  p.H = c->H;
  p.Hkv = c->Hkv;
  p.D = c->D;
  p.F = c->F;
  p.S_max = c->S;
  p.eps = c->a.norm_eps;
  p.attn_norm = reinterpret_cast<const bf16*>(Ly.attn_norm);
  p.ffn_norm = reinterpret_cast<const bf16*>(Ly.ffn_norm);
  p.h = h;
  p.q = reinterpret_cast<bf16*>(c->q);
  p.o = reinterpret_cast<bf16*>(c->o);
  p.g = reinterpret_cast<bf16*>(c->g);
  p.cache_k = reinterpret_cast<bf16*>(Ly.cache_k);
  p.cache_v = reinterpret_cast<bf16*>(Ly.cache_v);
  p.rope = c->rope;
  p.start_pos = sp_dev;
  p.sp_scalar = sp_host;
  p.part = c->part;
  p.counters = c->counters;
  p.ssq = c->ssq;
  p.gbar = c->gbar;
  p.err = c->err;
  p.hpc = pl.hpc;
  p.CK = pl.CK;
  p.max_chunks = pl.max_chunks;
  p.norm_local = pl.norm_local ? 1 : 0;
  const CUtensorMap maps[6] = {Ly.map_w[0], Ly.map_w[1], Ly.map_w[2], Ly.map_w[3], Ly.map_k, Ly.map_v};
  const cudaError_t e = launch_decode_block(maps, p, pl.grid, st);
  // a grid that cannot be resident at once is refused before anything runs
  if (e == cudaErrorCooperativeLaunchTooLarge) return LLAMA_ERR_INVALID_ARGS;
  return e == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

// Which decode attention kernel a call runs (both compute the same attention).
// AUTO takes the stream-K split once the call can hold at least 8 key tiles per
// SM (the longest history counted for every unit). Measured on B200: the
// LLaMA-2-70B layer at batch 16 x 4096 keys runs 0.343 ms per step against
// 0.360 chunked, the LLaMA-3-8B ragged batch-32 decode 436 ms per 64 steps
// against 446; a batch-1 LLaMA-7B layer over ~600 keys (about 2 tiles per SM)
// runs 90.8 us against 89.2 chunked. AUTO keeps groups of up to 8 query heads
// per CTA (the configurations timed above); 16 runs when chosen explicitly.
bool use_stream_k(int mode, const DecodeSkPlan& sk, int max_len, int num_sms) {
  if (mode != LLAMA_ATTN_AUTO) return mode == LLAMA_ATTN_STREAMK;
  const long long w_max = (long long)sk.units * ((max_len + 63) / 64);
  return sk.hpc <= 8 && w_max >= 8LL * num_sms;
}

int run_block(llama_ctx* c, int layer, float* h, int B, int T, const int* sp_dev, int sp_host, cudaStream_t st) {
  Layer& Ly = c->layers[layer];
  const int M = B * T;
  const int HD = c->H * c->D;
  int r;
  if (T == 1 && c->decode_mode == LLAMA_DECODE_PERSISTENT) {
    if (!c->bf16 || !c->gbar) return LLAMA_ERR_INVALID_ARGS;
    r = run_block_persistent(c, layer, h, B, sp_dev, sp_host, st);
    return r == 1 ? LLAMA_ERR_INVALID_ARGS : r;
  }
  const bool fnorm = fuse_norm(c, M);
  if (!fnorm && (c->bf16 ? launch_rmsnorm<bf16>(h, Ly.attn_norm, c->xn, M, c->dim, c->a.norm_eps, 1, 0, st)
                         : launch_rmsnorm<float>(h, Ly.attn_norm, c->xn, M, c->dim, c->a.norm_eps, 1, 0, st)) !=
                    cudaSuccess)
    return LLAMA_ERR_CUDA;

  EpiParams e = epi_base(c, EPI_QKV_ROPE, M, c->n_qkv);
  e.q_out = c->q;
  e.cache_k = Ly.cache_k;
  e.cache_v = Ly.cache_v;
  e.rope = c->rope;
  e.start_pos = sp_dev;
  e.start_pos_scalar = sp_host;
  e.T = T;
  e.H = c->H;
  e.Hkv = c->Hkv;
  e.D = c->D;
  e.S_max = c->S;
  if ((r = gemm(c, c->xn, Ly.wqkv, &Ly.map_w[0], M, c->n_qkv, c->dim, e, st, fnorm ? h : nullptr,
                fnorm ? Ly.attn_norm : nullptr)))
    return r;

  cudaError_t ce;
  if (!c->bf16) {
    ce = launch_attn_simple<float>(c->q, Ly.cache_k, Ly.cache_v, c->o, sp_dev, sp_host, B, T, c->H, c->Hkv, c->D,
                                   c->S, st);
  } else if (T == 1) {
    const int max_len = sp_dev ? c->S : sp_host + 1;
    DecodeSkPlan sk = plan_decode_sk(B, c->H, c->Hkv, c->D, max_len, c->num_sms);
    if (!sp_dev) align_decode_sk_uniform(sk, max_len, c->num_sms);
    if (c->attn_mode == LLAMA_ATTN_STREAMK && !sk.ok) return LLAMA_ERR_INVALID_ARGS;
    if (sk.ok && use_stream_k(c->attn_mode, sk, max_len, c->num_sms)) {
      if (sk.part_floats > c->part_floats || sk.units > c->counters_n) return LLAMA_ERR_INVALID_ARGS;
      ce = launch_attn_decode_sk(Ly.map_k, Ly.map_v, c->q, c->o, c->part, c->counters, sp_dev, sp_host, B, c->H,
                                 c->Hkv, c->D, c->S, sk, c->err, st);
    } else {
      DecodePlan p = plan_decode(B, c->H, c->Hkv, c->S, max_len, c->num_sms);
      if (p.part_floats > c->part_floats) return LLAMA_ERR_INVALID_ARGS;
      if (B * c->Hkv * (c->n_rep / p.hpc) > c->counters_n) return LLAMA_ERR_INVALID_ARGS;
      ce = launch_attn_decode(Ly.map_k, Ly.map_v, c->q, c->o, c->part, c->counters, sp_dev, sp_host, B, c->H,
                              c->Hkv, c->D, c->S, p, c->err, st);
    }
  } else {
    ce = launch_attn_prefill_tc(Ly.map_k, Ly.map_v, c->q, c->o, sp_dev, sp_host, B, T, c->H, c->Hkv, c->D, c->S,
                                c->err, st);
  }
  if (ce != cudaSuccess) return LLAMA_ERR_CUDA;

  e = epi_base(c, EPI_RESIDUAL, M, c->dim);
  e.out = h;
  e.ld_out = c->dim;
  if ((r = gemm(c, c->o, Ly.wo, &Ly.map_w[1], M, c->dim, HD, e, st))) return r;

  if (!fnorm && (c->bf16 ? launch_rmsnorm<bf16>(h, Ly.ffn_norm, c->xn, M, c->dim, c->a.norm_eps, 1, 0, st)
                         : launch_rmsnorm<float>(h, Ly.ffn_norm, c->xn, M, c->dim, c->a.norm_eps, 1, 0, st)) !=
                    cudaSuccess)
    return LLAMA_ERR_CUDA;

  e = epi_base(c, EPI_SWIGLU, M, 2 * c->F);
  e.g_out = c->g;
  if ((r = gemm(c, c->xn, Ly.w13, &Ly.map_w[2], M, 2 * c->F, c->dim, e, st, fnorm ? h : nullptr,
                fnorm ? Ly.ffn_norm : nullptr)))
    return r;

  e = epi_base(c, EPI_RESIDUAL, M, c->dim);
  e.out = h;
  e.ld_out = c->dim;
  return gemm(c, c->g, Ly.w2, &Ly.map_w[3], M, c->dim, c->F, e, st);
}

// embedding -> blocks -> final norm -> LM head
// col (device, optional; then T = 1): the tokens are column *col of `tokens`
// and sit at position *col; the embedding writes those positions to sp_dev.
int run_model(llama_ctx* c, const int32_t* tokens, int tok_stride, int B, int T, const int* sp_dev, int sp_host,
              float* logits, int all_positions, cudaStream_t st, const int* col = nullptr) {
  if (!c->head_set) return LLAMA_ERR_NOT_READY;
  for (int l = 0; l < c->L; ++l)
    if (!c->layers[l].set) return LLAMA_ERR_NOT_READY;
  const int M = B * T;
  int r;
  if ((r = reserve(c, M))) return r;
  int* pos_out = col ? const_cast<int*>(sp_dev) : nullptr;
  if ((c->bf16 ? launch_embed<bf16>(tokens, c->tok_emb, c->h, M, c->dim, c->V, T, tok_stride, c->err, st, col, pos_out)
               : launch_embed<float>(tokens, c->tok_emb, c->h, M, c->dim, c->V, T, tok_stride, c->err, st, col,
                                     pos_out)) != cudaSuccess)
    return LLAMA_ERR_CUDA;
  for (int l = 0; l < c->L; ++l)
    if ((r = run_block(c, l, c->h, B, T, sp_dev, sp_host, st))) return r;
  const int rows = all_positions ? M : B;
  const int stride = all_positions ? 1 : T;
  const int offset = all_positions ? 0 : T - 1;
  if ((c->bf16 ? launch_rmsnorm<bf16>(c->h, c->final_norm, c->xn, rows, c->dim, c->a.norm_eps, stride, offset, st)
               : launch_rmsnorm<float>(c->h, c->final_norm, c->xn, rows, c->dim, c->a.norm_eps, stride, offset,
                                       st)) != cudaSuccess)
    return LLAMA_ERR_CUDA;
  EpiParams e = epi_base(c, EPI_STORE_F32, rows, c->V);
  e.out = logits;
  e.ld_out = c->V;
  return gemm(c, c->xn, c->output, &c->map_out, rows, c->V, c->dim, e, st);
}

int check_ctx_call(llama_ctx* c, int B, int T) {
  if (!c) return LLAMA_ERR_INVALID_ARGS;
  if (B < 1 || B > c->Bm || T < 1) return LLAMA_ERR_INVALID_ARGS;
  if (cudaSetDevice(c->device) != cudaSuccess) return LLAMA_ERR_CUDA;
  return LLAMA_OK;
}

// private workspace of llama_linear
float* g_lin_part = nullptr;
size_t g_lin_part_floats = 0;
int* g_lin_counters = nullptr;
int g_lin_counters_n = 0;
int* g_lin_err = nullptr;
GemmSplitWs g_lin_split;  // the CTA-pair GEMM's k-split scratch (grown to the call's tiles)
int g_lin_dev = -1;  // device of the private workspace (the first call's)

}  // namespace

extern "C" {

int llama_ffn_hidden(const llama_args* a) {
  if (!a) return LLAMA_ERR_INVALID_ARGS;
  return ffn_hidden(a);
}

int llama_create(const llama_args* args, llama_ctx** out) {
  if (!args || !out) return LLAMA_ERR_INVALID_ARGS;
  *out = nullptr;
  llama_args a = *args;
  if (a.n_kv_heads <= 0) a.n_kv_heads = a.n_heads;
  if (a.dim <= 0 || a.n_layers <= 0 || a.n_heads <= 0 || a.max_batch_size <= 0 || a.max_seq_len <= 0 ||
      a.vocab_size < 0 || a.multiple_of <= 0 || !(a.norm_eps >= 0.f) || !(a.rope_theta > 0.f))
    return LLAMA_ERR_INVALID_ARGS;
  if (a.dtype != LLAMA_FP32 && a.dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARGS;
  if (a.rope_half_split != 0 && a.rope_half_split != 1) return LLAMA_ERR_INVALID_ARGS;
  if (a.dim % a.n_heads || a.n_heads % a.n_kv_heads || a.dim % 64) return LLAMA_ERR_INVALID_ARGS;
  const int D = a.dim / a.n_heads;
  if (D != 64 && D != 128) return LLAMA_ERR_INVALID_ARGS;
  const int n_rep = a.n_heads / a.n_kv_heads;
  const int F = ffn_hidden(&a);
  if (F < 0 || F % 64) return LLAMA_ERR_INVALID_ARGS;
  if (a.dtype == LLAMA_FP32 && (size_t)(a.max_seq_len + D) * 4 > 200 * 1024) return LLAMA_ERR_INVALID_ARGS;
  if (a.vocab_size % 8) return LLAMA_ERR_INVALID_ARGS;

  llama_ctx* c = new llama_ctx();
  c->a = a;
  c->bf16 = a.dtype == LLAMA_BF16;
  c->half_split = a.rope_half_split == 1;
  c->esz = c->bf16 ? 2 : 4;
  c->dim = a.dim;
  c->H = a.n_heads;
  c->Hkv = a.n_kv_heads;
  c->D = D;
  c->n_rep = n_rep;
  c->F = F;
  c->V = a.vocab_size;
  c->S = a.max_seq_len;
  c->Bm = a.max_batch_size;
  c->L = a.n_layers;
  c->n_qkv = (a.n_heads + 2 * a.n_kv_heads) * D;
  cudaGetDevice(&c->device);
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  c->layers.resize(a.n_layers);

  auto fail = [&](int code) {
    llama_destroy(c);
    return code;
  };
  int r;
  const size_t es = c->esz;
  const size_t wsz = (weight_elems(c, c->n_qkv, c->dim) + weight_elems(c, c->dim, (size_t)c->H * D) +
                      weight_elems(c, 2 * (size_t)F, c->dim) + weight_elems(c, c->dim, F)) * es;
  const size_t cache_elems = (size_t)c->Bm * c->Hkv * c->S * D;
  for (int l = 0; l < c->L; ++l) {
    Layer& Ly = c->layers[l];
    void* blob;
    if ((r = alloc(&blob, wsz + 2 * round256((size_t)c->dim * es)))) return fail(r);
    uint8_t* p = reinterpret_cast<uint8_t*>(blob);
    Ly.wqkv = p;
    p += weight_elems(c, c->n_qkv, c->dim) * es;
    Ly.wo = p;
    p += weight_elems(c, c->dim, (size_t)c->H * D) * es;
    Ly.w13 = p;
    p += weight_elems(c, 2 * (size_t)F, c->dim) * es;
    Ly.w2 = p;
    p += weight_elems(c, c->dim, F) * es;
    Ly.attn_norm = p;
    p += round256((size_t)c->dim * es);
    Ly.ffn_norm = p;
    if ((r = alloc(&Ly.cache_k, cache_elems * es))) return fail(r);
    if ((r = alloc(&Ly.cache_v, cache_elems * es))) return fail(r);
    if (cudaMemset(Ly.cache_k, 0, cache_elems * es) != cudaSuccess) return fail(LLAMA_ERR_CUDA);
    if (cudaMemset(Ly.cache_v, 0, cache_elems * es) != cudaSuccess) return fail(LLAMA_ERR_CUDA);
    if (c->bf16) {
      const uint64_t rows = (uint64_t)c->Bm * c->Hkv * c->S;
      if (!make_tmap_bf16(&Ly.map_k, Ly.cache_k, rows, D, 64) || !make_tmap_bf16(&Ly.map_v, Ly.cache_v, rows, D, 64))
        return fail(LLAMA_ERR_CUDA);
      if (!make_tmap_weights(&Ly.map_w[0], Ly.wqkv, 1, c->n_qkv, c->dim, 128) ||
          !make_tmap_weights(&Ly.map_w[1], Ly.wo, 1, c->dim, c->H * D, 128) ||
          !make_tmap_weights(&Ly.map_w[2], Ly.w13, 1, 2 * F, c->dim, 128) ||
          !make_tmap_weights(&Ly.map_w[3], Ly.w2, 1, c->dim, F, 128))
        return fail(LLAMA_ERR_CUDA);
    }
  }
  if (c->V > 0) {
    if ((r = alloc(&c->tok_emb, (size_t)c->V * c->dim * es))) return fail(r);
    if ((r = alloc(&c->final_norm, round256((size_t)c->dim * es)))) return fail(r);
    if ((r = alloc(&c->output, weight_elems(c, c->V, c->dim) * es))) return fail(r);
    if (c->bf16 && !make_tmap_weights(&c->map_out, c->output, 1, c->V, c->dim, 128)) return fail(LLAMA_ERR_CUDA);
  }
  std::vector<float2> rt = rope_table(D, 2 * c->S, (double)a.rope_theta);
  if ((r = alloc(reinterpret_cast<void**>(&c->rope), rt.size() * sizeof(float2)))) return fail(r);
  if (cudaMemcpy(c->rope, rt.data(), rt.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(LLAMA_ERR_CUDA);
  if ((r = alloc(reinterpret_cast<void**>(&c->err), sizeof(int)))) return fail(r);
  cudaMemset(c->err, 0, sizeof(int));

  // scratch: GEMV split-K partials for up to 32 tokens and decode-attention partials
  if (c->bf16) {
    const int mt = 32;  // the GEMV path serves any call of up to 32 tokens (B * T)
    const int Ns[5] = {c->n_qkv, c->dim, 2 * F, c->dim, c->V};
    const int Ks[5] = {c->dim, c->H * D, c->dim, F, c->dim};
    size_t need = 0;
    int rbs = 0;
    for (int i = 0; i < 5; ++i) {
      if (Ns[i] <= 0) continue;
      for (int m = 1; m <= mt; ++m) {
        GemvPlan p = plan_gemv(m, Ns[i], Ks[i], c->num_sms);
        if (p.part_floats > need) need = p.part_floats;
        if (p.row_blocks > rbs) rbs = p.row_blocks;
      }
    }
    const size_t dec = (size_t)c->Bm * c->H * ((c->S + 127) / 128) * (128 + 2);
    if (dec > need) need = dec;
    for (int b = 1; b <= c->Bm; ++b) {  // the stream-K decode attention's partials
      DecodeSkPlan sk = plan_decode_sk(b, c->H, c->Hkv, D, c->S, c->num_sms);
      if (sk.ok && sk.part_floats > need) need = sk.part_floats;
    }
    // the persistent decode kernel, for every batch it serves
    for (int m = 1; m <= c->Bm && m <= 32; ++m) {
      DecodeBlockPlan pl = plan_decode_block(m, c->dim, c->H, c->Hkv, D, F, c->S, c->S, c->num_sms);
      if (!pl.ok) continue;
      if (pl.part_floats > need) need = pl.part_floats;
      if (pl.counters > rbs) rbs = pl.counters;
    }
    c->part_floats = need;
    if ((r = alloc(reinterpret_cast<void**>(&c->part), need * sizeof(float)))) return fail(r);
    if (rbs < c->Bm * c->H) rbs = c->Bm * c->H;  // decode attention: one counter per (sequence, head group)
    c->counters_n = rbs;
    if ((r = alloc(reinterpret_cast<void**>(&c->counters), (size_t)rbs * sizeof(int)))) return fail(r);
    cudaMemset(c->counters, 0, (size_t)rbs * sizeof(int));
    if ((r = alloc(reinterpret_cast<void**>(&c->gbar), kGbarBytes))) return fail(r);
    cudaMemset(c->gbar, 0, kGbarBytes);
    const int bm = c->Bm < 32 ? c->Bm : 32;
    if ((r = alloc(reinterpret_cast<void**>(&c->ssq), (size_t)(c->dim / 64) * bm * sizeof(float)))) return fail(r);
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(LLAMA_ERR_CUDA);
  *out = c;
  return LLAMA_OK;
}

void llama_destroy(llama_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  for (Layer& Ly : c->layers) {
    release(Ly.wqkv);
    release(Ly.cache_k);
    release(Ly.cache_v);
  }
  release(c->tok_emb);
  release(c->final_norm);
  release(c->output);
  release(reinterpret_cast<void*&>(c->rope));
  release(reinterpret_cast<void*&>(c->err));
  release(reinterpret_cast<void*&>(c->h));
  release(c->xn);
  release(c->q);
  release(c->o);
  release(c->g);
  release(reinterpret_cast<void*&>(c->part));
  release(reinterpret_cast<void*&>(c->split.ws));
  release(reinterpret_cast<void*&>(c->split.sync));
  release(reinterpret_cast<void*&>(c->counters));
  release(reinterpret_cast<void*&>(c->gbar));
  release(reinterpret_cast<void*&>(c->ssq));
  release(reinterpret_cast<void*&>(c->gen_logits));
  release(reinterpret_cast<void*&>(c->gen_probs));
  release(reinterpret_cast<void*&>(c->gen_state));
  if (c->gen_exec) cudaGraphExecDestroy(c->gen_exec);
  delete c;
}

int llama_set_layer(llama_ctx* c, int layer, const void* wq, const void* wk, const void* wv, const void* wo,
                    const void* w1, const void* w2, const void* w3, const void* attn_norm, const void* ffn_norm) {
  if (!c || layer < 0 || layer >= c->L) return LLAMA_ERR_INVALID_ARGS;
  if (!wq || !wk || !wv || !wo || !w1 || !w2 || !w3 || !attn_norm || !ffn_norm) return LLAMA_ERR_INVALID_ARGS;
  for (const void* q : {wq, wk, wv, wo, w1, w2, w3})
    if (reinterpret_cast<uintptr_t>(q) % 16) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  Layer& Ly = c->layers[layer];
  const size_t es = c->esz;
  const size_t qb = (size_t)c->H * c->D * c->dim * es, kb = (size_t)c->Hkv * c->D * c->dim * es;
  // Row-major packing happens in place in fp32 mode; in bf16 mode it goes to a
  // temporary buffer from which the tiles are cut (tile_weights).
  void* tmp = nullptr;
  if (c->bf16) {
    const size_t n = std::max((size_t)c->n_qkv, 2 * (size_t)c->F) * c->dim * es;
    int r;
    if ((r = alloc(&tmp, n))) return r;
  }
  auto done = [&](int code) {
    if (tmp) {
      cudaDeviceSynchronize();
      release(tmp);
    }
    return code;
  };
#define CKT(call)                                             \
  do {                                                        \
    if ((call) != cudaSuccess) return done(LLAMA_ERR_CUDA);   \
  } while (0)
  uint8_t* p = reinterpret_cast<uint8_t*>(c->bf16 ? tmp : Ly.wqkv);
  if (c->half_split) {  // rotate interleaved pairs on rows permuted from the half-split order
    if (c->bf16) {
      launch_rope_rows_to_interleaved<bf16>(wq, p, c->H, c->D, c->dim, 0);
      launch_rope_rows_to_interleaved<bf16>(wk, p + qb, c->Hkv, c->D, c->dim, 0);
    } else {
      launch_rope_rows_to_interleaved<float>(wq, p, c->H, c->D, c->dim, 0);
      launch_rope_rows_to_interleaved<float>(wk, p + qb, c->Hkv, c->D, c->dim, 0);
    }
    CKT(cudaGetLastError());
  } else {
    CKT(cudaMemcpy(p, wq, qb, cudaMemcpyDeviceToDevice));
    CKT(cudaMemcpy(p + qb, wk, kb, cudaMemcpyDeviceToDevice));
  }
  CKT(cudaMemcpy(p + qb + kb, wv, kb, cudaMemcpyDeviceToDevice));
  CKT(cudaMemcpy(Ly.attn_norm, attn_norm, (size_t)c->dim * es, cudaMemcpyDeviceToDevice));
  CKT(cudaMemcpy(Ly.ffn_norm, ffn_norm, (size_t)c->dim * es, cudaMemcpyDeviceToDevice));
  if (c->bf16) {
    launch_tile_weights(tmp, Ly.wqkv, c->n_qkv, c->dim, 0);
    launch_tile_weights(wo, Ly.wo, c->dim, c->H * c->D, 0);
    launch_tile_weights(w2, Ly.w2, c->dim, c->F, 0);
    launch_pack_w13<bf16>(w1, w3, tmp, c->F, c->dim, 0);  // after the wqkv tiles have been cut (same stream)
    launch_tile_weights(tmp, Ly.w13, 2 * c->F, c->dim, 0);
  } else {
    CKT(cudaMemcpy(Ly.wo, wo, (size_t)c->dim * c->H * c->D * es, cudaMemcpyDeviceToDevice));
    CKT(cudaMemcpy(Ly.w2, w2, (size_t)c->dim * c->F * es, cudaMemcpyDeviceToDevice));
    launch_pack_w13<float>(w1, w3, Ly.w13, c->F, c->dim, 0);
  }
  CKT(cudaGetLastError());
  CKT(cudaDeviceSynchronize());
#undef CKT
  Ly.set = true;
  return done(LLAMA_OK);
}

int llama_set_embed_norm_head(llama_ctx* c, const void* tok, const void* norm, const void* output) {
  if (!c || c->V <= 0 || !tok || !norm || !output) return LLAMA_ERR_INVALID_ARGS;
  if (reinterpret_cast<uintptr_t>(output) % 16) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  const size_t es = c->esz;
  CK(cudaMemcpy(c->tok_emb, tok, (size_t)c->V * c->dim * es, cudaMemcpyDeviceToDevice));
  CK(cudaMemcpy(c->final_norm, norm, (size_t)c->dim * es, cudaMemcpyDeviceToDevice));
  if (c->bf16) {
    launch_tile_weights(output, c->output, c->V, c->dim, 0);
  } else {
    CK(cudaMemcpy(c->output, output, (size_t)c->V * c->dim * es, cudaMemcpyDeviceToDevice));
  }
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  c->head_set = true;
  return LLAMA_OK;
}

int llama_reserve(llama_ctx* c, int max_tokens) {
  if (!c || max_tokens < 1) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  return reserve(c, max_tokens);
}

int llama_forward(llama_ctx* c, const int32_t* tokens, int B, int T, int start_pos, float* logits, int all_positions,
                  void* stream) {
  int r;
  if ((r = check_ctx_call(c, B, T))) return r;
  if (!tokens || !logits || start_pos < 0 || (long)start_pos + T > c->S) return LLAMA_ERR_INVALID_ARGS;
  return run_model(c, tokens, T, B, T, nullptr, start_pos, logits, all_positions, S_(stream));
}

int llama_forward_ragged(llama_ctx* c, const int32_t* tokens, const int32_t* start_pos, int B, float* logits,
                         void* stream) {
  int r;
  if ((r = check_ctx_call(c, B, 1))) return r;
  if (!tokens || !start_pos || !logits) return LLAMA_ERR_INVALID_ARGS;
  return run_model(c, tokens, 1, B, 1, start_pos, 0, logits, 1, S_(stream));
}

int llama_block_forward(llama_ctx* c, int layer, float* h, int B, int T, const int32_t* start_pos_dev,
                        int host_start_pos, void* stream) {
  int r;
  if ((r = check_ctx_call(c, B, T))) return r;
  if (!h || layer < 0 || layer >= c->L) return LLAMA_ERR_INVALID_ARGS;
  if (!c->layers[layer].set) return LLAMA_ERR_NOT_READY;
  if (!start_pos_dev && (host_start_pos < 0 || (long)host_start_pos + T > c->S)) return LLAMA_ERR_INVALID_ARGS;
  if ((r = reserve(c, B * T))) return r;
  return run_block(c, layer, h, B, T, start_pos_dev, host_start_pos, S_(stream));
}

int llama_generate(llama_ctx* c, int32_t* tokens, const uint8_t* prompt_mask, int B, int total_len,
                   int min_prompt_len, float temperature, float top_p, const float* uniforms, void* stream) {
  int r;
  if ((r = check_ctx_call(c, B, 1))) return r;
  if (!tokens || !prompt_mask || c->V <= 0) return LLAMA_ERR_INVALID_ARGS;
  if (min_prompt_len < 1 || total_len > c->S || min_prompt_len > total_len) return LLAMA_ERR_INVALID_ARGS;
  const bool greedy = !(temperature > 0.f);
  if (!greedy && (!uniforms || !(top_p > 0.f) || !(top_p <= 1.f))) return LLAMA_ERR_INVALID_ARGS;
  if (!c->gen_logits) {
    const size_t n = (size_t)c->Bm * c->V * sizeof(float);
    if ((r = alloc(reinterpret_cast<void**>(&c->gen_logits), n))) return r;
    if ((r = alloc(reinterpret_cast<void**>(&c->gen_probs), n))) return r;
    if ((r = alloc(reinterpret_cast<void**>(&c->gen_state), (size_t)(1 + c->Bm) * sizeof(int)))) return r;
  }
  if ((r = reserve(c, B * min_prompt_len))) return r;
  if (c->gen_exec) {  // the previous call's graph: let its launches finish, then release it
    cudaStreamSynchronize(c->gen_exec_stream);
    cudaGraphExecDestroy(c->gen_exec);
    c->gen_exec = nullptr;
  }
  cudaStream_t st = S_(stream);
  const float* uni = greedy ? nullptr : uniforms;
  // Transformer.forward(tokens[:, prev:cur], prev) with last-position logits,
  // then the next token unless the sequence's prompt still covers position cur
  auto host_step = [&](int prev, int cur) -> int {
    int rr;
    if ((rr = run_model(c, tokens + prev, total_len, B, cur - prev, nullptr, prev, c->gen_logits, 0, st))) return rr;
    return launch_sample(c->gen_logits, B, c->V, temperature, top_p, uni ? uni + (size_t)cur * B : nullptr,
                         c->gen_probs, tokens + cur, total_len, prompt_mask + cur, total_len, st) == cudaSuccess
               ? LLAMA_OK
               : LLAMA_ERR_CUDA;
  };
  // One decode step whose column lives on the device (gen_state[0] = prev,
  // the column and position of the token fed in; the token chosen goes to
  // column prev + 1): the same kernels, so a CUDA graph of it replays unchanged.
  int* col = c->gen_state;
  int* pos = c->gen_state + 1;
  auto device_step = [&](cudaStream_t s) -> int {
    int rr;
    if ((rr = run_model(c, tokens, total_len, B, 1, pos, 0, c->gen_logits, 0, s, col))) return rr;
    if (launch_sample(c->gen_logits, B, c->V, temperature, top_p, uni ? uni + B : nullptr, c->gen_probs, tokens + 1,
                      total_len, prompt_mask + 1, total_len, s, col) != cudaSuccess)
      return LLAMA_ERR_CUDA;
    return launch_step_counter(col, 0, 1, s) == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
  };
  if (min_prompt_len >= total_len) return LLAMA_OK;
  // the prompt prefix, then one decode step per remaining position
  if ((r = host_step(0, min_prompt_len))) return r;
  const int first = min_prompt_len + 1, n_dec = total_len - first;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return LLAMA_ERR_CUDA;
  if (n_dec < 3 || cap != cudaStreamCaptureStatusNone) {
    // few steps, or the caller is capturing this stream itself: plain launches
    for (int cur = first; cur < total_len; ++cur)
      if ((r = host_step(cur - 1, cur))) return r;
    return LLAMA_OK;
  }
  // the first decode step runs directly (it also sets up every kernel it uses
  // on this device); the rest replay a graph captured from one step
  if (launch_step_counter(col, first - 1, 0, st) != cudaSuccess) return LLAMA_ERR_CUDA;
  if ((r = device_step(st))) return r;
  cudaStream_t cs;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return LLAMA_ERR_CUDA;
  cudaGraph_t graph = nullptr;
  r = LLAMA_OK;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    r = LLAMA_ERR_CUDA;
  } else {
    const int rs = device_step(cs);
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess || rs != LLAMA_OK) r = rs != LLAMA_OK ? rs : LLAMA_ERR_CUDA;
  }
  cudaStreamDestroy(cs);
  if (r == LLAMA_OK && cudaGraphInstantiate(&c->gen_exec, graph, 0) != cudaSuccess) r = LLAMA_ERR_CUDA;
  if (graph) cudaGraphDestroy(graph);
  if (r != LLAMA_OK) {
    c->gen_exec = nullptr;
    return r;
  }
  c->gen_exec_stream = st;
  for (int i = 1; i < n_dec; ++i)
    if (cudaGraphLaunch(c->gen_exec, st) != cudaSuccess) return LLAMA_ERR_CUDA;
  return LLAMA_OK;
}

int llama_kv_read(llama_ctx* c, int layer, void* k, void* v, void* stream) {
  if (!c || layer < 0 || layer >= c->L || !k || !v) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  Layer& Ly = c->layers[layer];
  if (c->bf16) {
    launch_kv_convert<bf16>(Ly.cache_k, k, c->Bm, c->S, c->Hkv, c->D, 1, c->half_split, S_(stream));
    launch_kv_convert<bf16>(Ly.cache_v, v, c->Bm, c->S, c->Hkv, c->D, 1, 0, S_(stream));
  } else {
    launch_kv_convert<float>(Ly.cache_k, k, c->Bm, c->S, c->Hkv, c->D, 1, c->half_split, S_(stream));
    launch_kv_convert<float>(Ly.cache_v, v, c->Bm, c->S, c->Hkv, c->D, 1, 0, S_(stream));
  }
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int llama_kv_write(llama_ctx* c, int layer, const void* k, const void* v, void* stream) {
  if (!c || layer < 0 || layer >= c->L || !k || !v) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  Layer& Ly = c->layers[layer];
  if (c->bf16) {
    launch_kv_convert<bf16>(k, Ly.cache_k, c->Bm, c->S, c->Hkv, c->D, 0, c->half_split, S_(stream));
    launch_kv_convert<bf16>(v, Ly.cache_v, c->Bm, c->S, c->Hkv, c->D, 0, 0, S_(stream));
  } else {
    launch_kv_convert<float>(k, Ly.cache_k, c->Bm, c->S, c->Hkv, c->D, 0, c->half_split, S_(stream));
    launch_kv_convert<float>(v, Ly.cache_v, c->Bm, c->S, c->Hkv, c->D, 0, 0, S_(stream));
  }
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int llama_reset(llama_ctx* c) {
  if (!c) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  const size_t bytes = (size_t)c->Bm * c->Hkv * c->S * c->D * c->esz;
  for (Layer& Ly : c->layers) {
    CK(cudaMemset(Ly.cache_k, 0, bytes));
    CK(cudaMemset(Ly.cache_v, 0, bytes));
  }
  if (c->counters) CK(cudaMemset(c->counters, 0, (size_t)c->counters_n * sizeof(int)));
  if (c->gbar) CK(cudaMemset(c->gbar, 0, kGbarBytes));
  CK(cudaDeviceSynchronize());
  return LLAMA_OK;
}

int llama_set_decode_attention(llama_ctx* c, int mode) {
  if (!c || mode < LLAMA_ATTN_AUTO || mode > LLAMA_ATTN_STREAMK) return LLAMA_ERR_INVALID_ARGS;
  c->attn_mode = mode;
  return LLAMA_OK;
}

int llama_set_decode_linear_mma(int mode) {
  return set_gemv_mma(mode) == 0 ? LLAMA_OK : LLAMA_ERR_INVALID_ARGS;
}

int llama_set_decode_kernel(llama_ctx* c, int mode) {
  if (!c || mode < LLAMA_DECODE_AUTO || mode > LLAMA_DECODE_PERSISTENT) return LLAMA_ERR_INVALID_ARGS;
  c->decode_mode = mode;
  return LLAMA_OK;
}

int llama_get_error(llama_ctx* c, int* flags) {
  if (flags) *flags = 0;
  if (!c) return LLAMA_ERR_INVALID_ARGS;
  CK(cudaSetDevice(c->device));
  if (cudaDeviceSynchronize() != cudaSuccess) return LLAMA_ERR_CUDA;
  int f = 0;
  CK(cudaMemcpy(&f, c->err, sizeof(int), cudaMemcpyDeviceToHost));
  CK(cudaMemset(c->err, 0, sizeof(int)));
  if (flags) *flags = f;
  if (f & LLAMA_DEV_TIMEOUT) {
    // a wait that gave up can leave arrival counters mid-count: re-arm them
    if (c->counters) cudaMemset(c->counters, 0, (size_t)c->counters_n * sizeof(int));
    if (c->gbar) cudaMemset(c->gbar, 0, kGbarBytes);
    cudaDeviceSynchronize();
    return LLAMA_ERR_TIMEOUT;
  }
  if (f & LLAMA_DEV_POS_RANGE) return LLAMA_ERR_POS_RANGE;
  if (f & LLAMA_DEV_TOKEN_RANGE) return LLAMA_ERR_TOKEN_RANGE;
  return LLAMA_OK;
}

const char* llama_strerror(int code) {
  switch (code) {
    case LLAMA_OK: return "ok";
    case LLAMA_ERR_INVALID_ARGS: return "invalid arguments";
    case LLAMA_ERR_OOM: return "device out of memory";
    case LLAMA_ERR_CUDA: return "CUDA error";
    case LLAMA_ERR_NOT_READY: return "weights not set";
    case LLAMA_ERR_TOO_LARGE: return "size exceeds the fixed scratch of llama_linear_noalloc";
    case LLAMA_ERR_INTERNAL: return "an internal consistency check failed";
    case LLAMA_ERR_TOKEN_RANGE: return "token id outside [0, vocab_size)";
    case LLAMA_ERR_POS_RANGE: return "position outside [0, max_seq_len)";
    case LLAMA_ERR_TIMEOUT: return "a bounded device wait timed out";
    default: return "unknown error";
  }
}

int llama_sample(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                 int32_t* out, void* stream) {
  if (!logits || !out || B < 1 || V < 1) return LLAMA_ERR_INVALID_ARGS;
  const bool greedy = !(temperature > 0.f);
  if (!greedy && (!uniforms || !(top_p > 0.f) || !(top_p <= 1.f))) return LLAMA_ERR_INVALID_ARGS;
  static float* scratch = nullptr;
  static size_t scratch_n = 0;
  static int scratch_dev = -1;  // the scratch lives on the device of the first top-p call
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLAMA_ERR_CUDA;
  if (!greedy && scratch_dev >= 0 && dev != scratch_dev) return LLAMA_ERR_INVALID_ARGS;
  if (!greedy && scratch_n < (size_t)B * V) {
    scratch_dev = dev;
    cudaDeviceSynchronize();
    release(reinterpret_cast<void*&>(scratch));
    scratch_n = 0;
    if (alloc(reinterpret_cast<void**>(&scratch), (size_t)B * V * sizeof(float))) return LLAMA_ERR_OOM;
    scratch_n = (size_t)B * V;
  }
  return launch_sample(logits, B, V, temperature, top_p, uniforms, scratch, out, 1, nullptr, 0, S_(stream)) ==
                 cudaSuccess
             ? LLAMA_OK
             : LLAMA_ERR_CUDA;
}

int llama_selfcheck_plans(int M, int dim, int n_heads, int n_kv_heads, int ffn, int max_seq_len, int num_sms) {
  if (M < 1 || dim < 64 || n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads || dim % n_heads || ffn < 64 ||
      max_seq_len < 1 || num_sms < 1 || dim % 64 || ffn % 64)
    return LLAMA_ERR_INVALID_ARGS;
  const int D = dim / n_heads, n_qkv = (n_heads + 2 * n_kv_heads) * D;
  // the decode GEMV of every linear, for the tokens given
  if (M <= 32) {
    const int Ns[4] = {n_qkv, dim, 2 * ffn, dim};
    const int Ks[4] = {dim, n_heads * D, dim, ffn};
    for (int i = 0; i < 4; ++i)
      if (Ks[i] % 64 == 0 && !check_gemv_plan(M, Ns[i], Ks[i], num_sms)) return LLAMA_ERR_INTERNAL;
  }
  // the persistent decode kernel, with the workspace a context would hold
  DecodeBlockPlan pl = plan_decode_block(M, dim, n_heads, n_kv_heads, D, ffn, max_seq_len, max_seq_len, num_sms);
  if (pl.ok && !check_decode_block_plan(pl, M, n_heads, pl.part_floats, pl.counters)) return LLAMA_ERR_INTERNAL;
  // the prefill attention's head groups: whole heads, and 128 rows of whole positions
  {
    const int hp = prefill_heads_per_cta(n_heads / n_kv_heads);
    if (128 % hp || !check_decode_heads(n_heads, n_kv_heads, hp)) return LLAMA_ERR_INTERNAL;
  }
  // the chunked decode attention's head groups
  if (!check_decode_heads(n_heads, n_kv_heads, plan_decode(M, n_heads, n_kv_heads, max_seq_len, max_seq_len, num_sms).hpc))
    return LLAMA_ERR_INTERNAL;
  // the stream-K decode attention: ragged device positions (planned for max_seq_len) ...
  std::vector<int> pos(M);
  const int S = max_seq_len;
  DecodeSkPlan sk = plan_decode_sk(M, n_heads, n_kv_heads, D, S, num_sms);
  uint32_t lcg = 12345u + (uint32_t)M;
  for (int pattern = 0; pattern < 5; ++pattern) {
    for (int b = 0; b < M; ++b) {
      lcg = lcg * 1664525u + 1013904223u;
      pos[b] = pattern == 0 ? S - 1
             : pattern == 1 ? (int)(((long long)b * 977 + 13) % S)
             : pattern == 2 ? (b == 0 ? S - 1 : 0)
             : pattern == 3 ? 0
                            : (int)((lcg >> 8) % (uint32_t)S);
    }
    if (!check_decode_sk(sk, pos.data(), M, n_heads, n_kv_heads, D, S)) return LLAMA_ERR_INTERNAL;
  }
  // ... and one position for the whole batch (planned for that length)
  const int sps[5] = {0, 63, 64, S / 3, S - 1};
  for (int sp : sps) {
    DecodeSkPlan p1 = plan_decode_sk(M, n_heads, n_kv_heads, D, sp + 1, num_sms);
    std::fill(pos.begin(), pos.end(), sp);
    if (!check_decode_sk(p1, pos.data(), M, n_heads, n_kv_heads, D, S)) return LLAMA_ERR_INTERNAL;
    align_decode_sk_uniform(p1, sp + 1, num_sms);  // the grid such calls launch
    if (!check_decode_sk(p1, pos.data(), M, n_heads, n_kv_heads, D, S)) return LLAMA_ERR_INTERNAL;
  }
  return LLAMA_OK;
}

int llama_set_alloc_limit(uint64_t bytes) {
  std::lock_guard<std::mutex> lock(g_alloc_mu);
  g_alloc_limit = bytes;
  return LLAMA_OK;
}

uint64_t llama_allocated_bytes(void) {
  std::lock_guard<std::mutex> lock(g_alloc_mu);
  return g_alloc_total;
}

int llama_selftest_bounded_wait(int which, int* flags, double* seconds) {
  if (flags) *flags = 0;
  if (seconds) *seconds = 0.0;
  if (which != 0 && which != 1) return LLAMA_ERR_INVALID_ARGS;
  void* buf = nullptr;  // error word, elapsed time, 256-byte grid-barrier block
  int r;
  if ((r = alloc(&buf, 512))) return r;
  uint8_t* b = reinterpret_cast<uint8_t*>(buf);
  int* err = reinterpret_cast<int*>(b);
  unsigned long long* elapsed = reinterpret_cast<unsigned long long*>(b + 8);
  void* gbar = b + 256;
  int code = LLAMA_OK;
  if (cudaMemset(buf, 0, 512) != cudaSuccess) code = LLAMA_ERR_CUDA;
  if (code == LLAMA_OK) {
    const cudaError_t e = which == 0 ? launch_mbarrier_selftest(err, elapsed, 0)
                                     : launch_grid_barrier_selftest(gbar, err, elapsed, 0);
    if (e != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) code = LLAMA_ERR_CUDA;
  }
  int f = 0;
  unsigned long long ns = 0;
  if (code == LLAMA_OK && (cudaMemcpy(&f, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
                           cudaMemcpy(&ns, elapsed, sizeof(ns), cudaMemcpyDeviceToHost) != cudaSuccess))
    code = LLAMA_ERR_CUDA;
  release(buf);
  if (flags) *flags = f;
  if (seconds) *seconds = (double)ns * 1e-9;
  return code;
}

int llama_tile_weights(const void* w, void* out, int N, int K, void* stream) {
  if (!w || !out || N <= 0 || K <= 0 || K % 64) return LLAMA_ERR_INVALID_ARGS;
  if (reinterpret_cast<uintptr_t>(w) % 16 || reinterpret_cast<uintptr_t>(out) % 16) return LLAMA_ERR_INVALID_ARGS;
  launch_tile_weights(w, out, N, K, S_(stream));
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int llama_linear(const void* x, const void* w, float* y, int M, int N, int K, int dtype, int path, void* stream) {
  if (!x || !w || !y || M <= 0 || N <= 0 || K <= 0 || N % 8 || K % 8) return LLAMA_ERR_INVALID_ARGS;
  if (dtype != LLAMA_FP32 && dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARGS;
  const int tiled = (path & LLAMA_WEIGHTS_TILED) ? 1 : 0;
  path &= ~LLAMA_WEIGHTS_TILED;
  if (tiled && (dtype != LLAMA_BF16 || K % 64 || path == LLAMA_PATH_SIMT)) return LLAMA_ERR_INVALID_ARGS;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (g_lin_dev >= 0 && dev != g_lin_dev) return LLAMA_ERR_INVALID_ARGS;  // the workspace is on another device
  g_lin_dev = dev;
  if (path == LLAMA_PATH_AUTO)
    path = dtype == LLAMA_FP32 ? LLAMA_PATH_SIMT : (M <= 32 && K % 64 == 0 ? LLAMA_PATH_GEMV : LLAMA_PATH_TCGEN05);
  if (!g_lin_err) {
    if (alloc(reinterpret_cast<void**>(&g_lin_err), sizeof(int))) return LLAMA_ERR_OOM;
    cudaMemset(g_lin_err, 0, sizeof(int));
  }
  EpiParams e;
  std::memset(&e, 0, sizeof(e));
  e.kind = EPI_STORE_F32;
  e.M = M;
  e.N = N;
  e.out = y;
  e.ld_out = N;
  e.err = g_lin_err;
  cudaStream_t st = S_(stream);
  switch (path) {
    case LLAMA_PATH_SIMT:
      if (dtype == LLAMA_FP32)
        launch_gemm_simt<float>(x, w, M, N, K, e, st);
      else
        launch_gemm_simt<bf16>(x, w, M, N, K, e, st);
      break;
    case LLAMA_PATH_GEMV: {
      if (dtype != LLAMA_BF16 || M > 32 || K % 64) return LLAMA_ERR_INVALID_ARGS;
      GemvPlan p = plan_gemv(M, N, K, sms);
      if (p.part_floats > g_lin_part_floats) {
        cudaDeviceSynchronize();
        release(reinterpret_cast<void*&>(g_lin_part));
        g_lin_part_floats = 0;
        if (alloc(reinterpret_cast<void**>(&g_lin_part), p.part_floats * sizeof(float))) return LLAMA_ERR_OOM;
        g_lin_part_floats = p.part_floats;
      }
      if (p.row_blocks > g_lin_counters_n) {
        cudaDeviceSynchronize();
        release(reinterpret_cast<void*&>(g_lin_counters));
        g_lin_counters_n = 0;
        if (alloc(reinterpret_cast<void**>(&g_lin_counters), (size_t)p.row_blocks * sizeof(int))) return LLAMA_ERR_OOM;
        cudaMemset(g_lin_counters, 0, (size_t)p.row_blocks * sizeof(int));
        g_lin_counters_n = p.row_blocks;
      }
      if (launch_gemv_bf16(x, w, tiled, M, N, K, p, g_lin_part, g_lin_counters, e, sms, st) != cudaSuccess)
        return LLAMA_ERR_CUDA;
      break;
    }
    case LLAMA_PATH_TCGEN05:
    {
      if (dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARGS;
      const int tiles = std::min(((M + 255) / 256) * ((N + 255) / 256), gemm_split_max_tiles(sms));
      if (tiled && tiles > g_lin_split.tiles) {
        cudaDeviceSynchronize();
        release(reinterpret_cast<void*&>(g_lin_split.ws));
        release(reinterpret_cast<void*&>(g_lin_split.sync));
        g_lin_split.tiles = 0;
        if (alloc(reinterpret_cast<void**>(&g_lin_split.ws), gemm_split_ws_floats(tiles) * sizeof(float)))
          return LLAMA_ERR_OOM;
        if (alloc(reinterpret_cast<void**>(&g_lin_split.sync), gemm_split_sync_ints(tiles) * sizeof(int)))
          return LLAMA_ERR_OOM;
        cudaMemset(g_lin_split.sync, 0, gemm_split_sync_ints(tiles) * sizeof(int));
        g_lin_split.tiles = tiles;
      }
      if (launch_gemm_tc(x, w, tiled, M, N, K, e, sms, st, nullptr, &g_lin_split) != cudaSuccess)
        return LLAMA_ERR_CUDA;
      break;
    }
    default:
      return LLAMA_ERR_INVALID_ARGS;
  }
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

}  // extern "C"
