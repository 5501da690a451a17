// Launchers of the library's kernels (host-side declarations).
#pragma once

#include <atomic>
#include <utility>

#include "common.cuh"

namespace llama {

// Launch with programmatic stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Opt a kernel in to `bytes` of dynamic shared memory on the current device,
// once per device (the attribute is per device; `done` is one bit per device
// ordinal, kept by the caller in a static).
template <typename... KArgs>
cudaError_t ensure_smem(void (*kernel)(KArgs...), size_t bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// elementwise.cu
template <typename T>
cudaError_t launch_embed(const int* tokens, const void* table, float* h, int n_tok, int dim, int vocab, int T_,
                         int tok_stride, int* err, cudaStream_t st, const int* col = nullptr, int* pos = nullptr);
cudaError_t launch_step_counter(int* col, int value, int add, cudaStream_t st);
template <typename T>
cudaError_t launch_rmsnorm(const float* h, const void* w, void* out, int rows, int dim, float eps,
                           int in_row_stride_T, int in_row_offset, cudaStream_t st);
template <typename T>
void launch_pack_w13(const void* w1, const void* w3, void* out, int F, int dim, cudaStream_t st);
template <typename T>
void launch_kv_convert(const void* src, void* dst, int Bm, int S, int Hkv, int D, int to_logical, int half_split,
                       cudaStream_t st);
template <typename T>
void launch_rope_rows_to_interleaved(const void* src, void* dst, int heads, int D, int dim, cudaStream_t st);
// [N][K] row-major bf16 -> [ceil(N/128)][K/64][128][64] tiles (rows past N zero); K % 64 == 0
void launch_tile_weights(const void* src, void* dst, int N, int K, cudaStream_t st);
__host__ __device__ constexpr size_t tiled_weight_elems(size_t N, size_t K) { return (N + 127) / 128 * 128 * K; }

// gemm_simt.cu
template <typename T>
void launch_gemm_simt(const void* A, const void* W, int M, int N, int K, const EpiParams& ep, cudaStream_t st);

// gemv.cu
struct GemvPlan {
  int row_blocks = 0, nk = 0, total = 0, grid = 1, S = 1;  // S = most CTAs sharing one row block
  size_t part_floats = 0;
};
GemvPlan plan_gemv(int M, int N, int K, int num_sms);
bool check_gemv_plan(int M, int N, int K, int num_sms);  // host walk of a plan (see gemv.cu)
// W: [N][K] row-major (tiled = 0) or the library's weight tiles (tiled = 1, tile_weights)
// wmap (optional): a tensor map of W encoded once by the caller (tiled layout, 128-row boxes); else encoded here
// h_norm (optional): X is not read; the kernel computes X = RMSNorm(h_norm) itself, h_norm [M][K] fp32 rows,
// w_norm [K] bf16, eps (the RMSNorm kernel's arithmetic); only where gemv_can_fuse_norm(M, K)
cudaError_t launch_gemv_bf16(const void* X, const void* W, int tiled, int M, int N, int K, const GemvPlan& p,
                             float* part, int* counters, const EpiParams& ep, int num_sms, cudaStream_t st,
                             const CUtensorMap* wmap = nullptr, const float* h_norm = nullptr,
                             const void* w_norm = nullptr, float eps = 0.f);
bool gemv_can_fuse_norm(int M, int K);
// LLAMA_GEMV_MMA_* for the 9..32-token calls (process-wide); -1 for another mode
int set_gemv_mma(int mode);

// gemm_tc.cu
bool make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_tmap_bf16_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                       uint32_t b1, uint32_t b2);
bool make_tmap_weights(CUtensorMap* map, const void* ptr, int tiled, uint64_t N, uint64_t K, uint32_t box_rows);
// Scratch of the CTA-pair GEMM's two-way k split, for up to `tiles` 256 x 256
// tiles: ws gemm_split_ws_floats(tiles) floats, sync gemm_split_sync_ints(tiles)
// ints, zeroed once (every launch leaves them zeroed).
struct GemmSplitWs {
  float* ws = nullptr;
  int* sync = nullptr;
  int tiles = 0;
};
size_t gemm_split_ws_floats(int tiles);
size_t gemm_split_sync_ints(int tiles);
int gemm_split_max_tiles(int num_sms);  // the largest tile count that can take the split
// bmap (optional, tiled B only): a tensor map of B encoded once by the caller (128-row boxes)
// split (optional): scratch that lets small-M calls split each pair tile's k range in two
cudaError_t launch_gemm_tc(const void* A, const void* B, int b_tiled, int M, int N, int K, const EpiParams& ep,
                           int num_sms, cudaStream_t st, const CUtensorMap* bmap = nullptr,
                           const GemmSplitWs* split = nullptr);

// Query heads one decode-attention CTA serves (one kv head's group of n_rep
// query heads, split into n_rep / hpc groups; an MMA row block holds 16): all of
// them up to 16, else 16 or 8 when one of them divides n_rep, else the largest
// divisor of n_rep below 16 (n_rep 20 -> 10, 17 -> 1), so every ratio the pages'
// repeat_kv allows is served.
inline int decode_heads_per_cta(int n_rep) {
  if (n_rep <= 16) return n_rep;
  if (n_rep % 16 == 0) return 16;
  if (n_rep % 8 == 0) return 8;
  int hpc = 15;
  while (n_rep % hpc) --hpc;
  return hpc;
}
// Query heads one prefill-attention CTA serves: its 128 MMA rows hold 128 / hpc
// positions x hpc heads, so hpc must divide 128 as well as n_rep: the largest
// power of two dividing n_rep, at most 8 (n_rep 6 -> 2, n_rep 3, 5, 7 -> 1).
inline int prefill_heads_per_cta(int n_rep) {
  int hpc = 1;
  while (hpc < 8 && n_rep % (2 * hpc) == 0) hpc *= 2;
  return hpc;
}
// Every query head of every kv head in exactly one group of the split above.
bool check_decode_heads(int H, int Hkv, int hpc);

// attention.cu
struct DecodePlan {
  int hpc = 1, CK = 256, max_chunks = 1;
  size_t part_floats = 0;
};
DecodePlan plan_decode(int B, int H, int Hkv, int S_max, int max_len, int num_sms);
cudaError_t launch_attn_decode(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                               int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int D, int S_max,
                               const DecodePlan& p, int* err, cudaStream_t st);
// attn_decode_sk.cu: the same decode attention with the key tiles of all
// (sequence, head group) units dealt out stream-K over two CTAs per SM
struct DecodeSkPlan {
  bool ok = false;  // shape served (B <= 1024, head_dim 64 or 128, 32-bit split arithmetic)
  int hpc = 1, grid = 1, units = 0;
  size_t part_floats = 0;
};
DecodeSkPlan plan_decode_sk(int B, int H, int Hkv, int D, int max_len, int num_sms);
// calls whose sequences all hold `len` keys: a grid of whole CTAs per unit where it pays (shrinks only)
void align_decode_sk_uniform(DecodeSkPlan& p, int len, int num_sms);
cudaError_t launch_attn_decode_sk(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                                  int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int D, int S_max,
                                  const DecodeSkPlan& p, int* err, cudaStream_t st);
bool check_decode_sk(const DecodeSkPlan& p, const int* start_pos, int B, int H, int Hkv, int D, int S_max);
// sample.cu
// col (optional, device): out, keep and the uniforms row are offset by column *col
cudaError_t launch_sample(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                          float* scratch, int32_t* out, int out_stride, const uint8_t* keep, int keep_stride,
                          cudaStream_t st, const int* col = nullptr);

// attn_tc.cu
cudaError_t launch_attn_prefill_tc(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o,
                                   const int* sp, int sp_scalar, int B, int T, int H, int Hkv, int D, int S_max,
                                   int* err, cudaStream_t st);
template <typename T>
cudaError_t launch_attn_simple(const void* q, const void* ck, const void* cv, void* o, const int* sp, int sp_scalar,
                               int B, int T_, int H, int Hkv, int D, int S_max, cudaStream_t st);


// decode_block.cu: one decode step of a whole block in one persistent launch
constexpr int DB_RING_STAGES = 9;                 // 16 KB weight tiles in flight per SM
constexpr uint32_t DB_AREA_BYTES = 64 * 1024;     // x slice of a linear / K,V tiles of the attention

struct DbLinear {  // one linear [N][K] as stream-K stages of 128 rows x 64 k, k cut into S slices
  int N = 0, K = 0, RB = 0, NK = 0, S = 1, total = 0;
};

struct DecodeBlockParams {
  DbLinear lin[4];  // wqkv, wo, w1|w3, w2
  int M, dim, H, Hkv, D, F, S_max;
  float eps;
  const bf16* attn_norm;
  const bf16* ffn_norm;
  float* h;          // [M][dim] fp32 residual stream, in/out
  bf16* q;           // [M][H*D]
  bf16* o;           // [M][H*D]
  bf16* g;           // [M][F]
  bf16* cache_k;     // this layer's cache [B_max][Hkv][S_max][D]
  bf16* cache_v;
  const float2* rope;
  const int* start_pos;  // [M] device positions, or nullptr -> sp_scalar
  int sp_scalar;
  float* part;       // partial tiles (linears) and chunk partials (attention)
  int* counters;     // self-resetting arrival counters
  float* ssq;        // [dim/128][M] sums of squares of h per 128-column block
  unsigned* gbar;    // grid barrier: one 64-bit arrival counter
  int* err;
  int hpc, CK, max_chunks;  // attention split
  int norm_local;    // 1: a linear's x slice is the whole row; RMSNorm statistics are computed where it is loaded
};

struct DecodeBlockPlan {
  bool ok = false;
  DbLinear lin[4];
  int grid = 1, hpc = 1, CK = 128, max_chunks = 1, counters = 0;
  bool norm_local = false;
  size_t part_floats = 0;
};
DecodeBlockPlan plan_decode_block(int M, int dim, int H, int Hkv, int D, int F, int S_max, int max_len,
                                  int num_sms);
// maps: wqkv, wo, w1|w3, w2 (128-row x 64-k boxes), then the layer's K and V caches (64-row x 64 boxes)
cudaError_t launch_decode_block(const CUtensorMap* maps, const DecodeBlockParams& p, int grid, cudaStream_t st);
size_t decode_block_smem(int M);
bool check_decode_block_plan(const DecodeBlockPlan& pl, int M, int H, size_t part_floats, int counters_n);
// failure-detection self-tests (selftest.cu, decode_block.cu): a bounded wait that nothing completes
cudaError_t launch_grid_barrier_selftest(void* gbar, int* err, unsigned long long* elapsed, cudaStream_t st);
cudaError_t launch_mbarrier_selftest(int* err, unsigned long long* elapsed, cudaStream_t st);

}  // namespace llama
