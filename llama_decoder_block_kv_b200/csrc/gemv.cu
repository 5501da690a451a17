// Decode GEMM for a handful of tokens (M <= 32): C[M][N] = X[M][K] * W[N][K]^T.
//
// At decode time every weight byte is read once per step and the token count
// is tiny, so this kernel is bound by HBM bandwidth, not by tensor throughput
// (the KV-cache section of "LLaMa-1/2/3 原理+源码——拆解" makes the same
// point: with the cache the bottleneck becomes memory access).
//
// Persistent stream-K kernel, at most one CTA per SM (see plan_gemv for the
// grid): the weight stages of all row blocks (128 rows x 64 k each) are dealt
// out as equal contiguous ranges. A
// producer warp streams its range's weight tiles together with the matching
// X tiles (8*MB tokens x 64 bf16) through a deep shared-memory ring with TMA
// (128-byte swizzle, no multicast), never pausing at row-block edges. The
// weights are either row-major or the library's tile layout (each stage one
// contiguous 16 KB block, see tile_weights_kernel); the shared-memory image
// of a stage is the same for both. Four
// consumer warps (32 weight rows each) read the tiles with ldmatrix into the
// warp-level bf16 tensor-core MMA, weights as the 16-row operand ("swap AB"):
// one MMA covers 16 weight rows x 8 tokens x 16 k.
//
// A row block that spans several CTAs' ranges gets one fp32 partial tile per
// CTA in a workspace and a per-row-block counter; the CTA that arrives last
// sums the partials in a fixed order (deterministic) and runs the epilogue,
// then re-zeroes the counter, so the workspace needs no clearing between
// launches. A row block inside one range goes straight to the epilogue.
//
// For decode calls of at most NORM_MAX_M tokens with K <= NORM_MAX_K the
// kernel can also compute its input X = RMSNorm(h) itself (the notes'
// RMSNorm.forward: fp32 statistics, the normalised value rounded to bf16,
// times the weight, rounded again), which takes the RMSNorm launch and the X
// round trip through memory off the decode step. The producer copies the norm
// weight into shared memory ahead of the ring's first weight tiles (plain
// loads issued beside those copies waited behind them for microseconds) and
// fetches only NORM_PREFETCH stages before the dependency wait; after it the
// consumer warps load all of their share of h at once, reduce the sums of
// squares across the CTA and keep the M normalised rows resident in shared
// memory for the whole K; the ring carries weight tiles only.
#include "kernels.cuh"

#include <algorithm>
#include <vector>

namespace llama {

namespace {
constexpr int RPC = 128;                   // weight rows per unit
constexpr int KB = 64;                     // k per ring stage (one 128-byte swizzle row)
constexpr uint32_t W_BYTES = RPC * KB * 2; // 16 KB
constexpr int OS = RPC + 4;                // row stride of the fp32 output staging tile
// A deep ring (~180 KB, 9-10 weight tiles in flight per SM): measured faster
// than a 104 KB ring that would let the next kernel's CTA share the SM.
constexpr size_t RING_BUDGET = 180 * 1024;

__host__ __device__ constexpr uint32_t x_bytes(int mb) { return 8u * mb * KB * 2; }
__host__ __device__ constexpr uint32_t stage_bytes(int mb) { return W_BYTES + x_bytes(mb); }
__host__ __device__ constexpr int stages(int mb) { return (int)(RING_BUDGET / stage_bytes(mb)); }
__host__ __device__ constexpr size_t gemv_smem(int mb) {
  return 1024 + (size_t)stages(mb) * stage_bytes(mb) + (size_t)8 * mb * OS * 4 + 2 * stages(mb) * 8 + 16;
}

constexpr int NORM_MAX_M = 4;
constexpr int NORM_MAX_K = 4096;
constexpr int NORM_CHUNKS = NORM_MAX_K / (128 * 4);  // float4 chunks of one row per consumer thread
// resident row stride in bytes: 16 bytes past a multiple of 128, so the rows
// an ldmatrix reads together sit in different banks
constexpr uint32_t NORM_XS = NORM_MAX_K * 2 + 16;
constexpr int NORM_STAGES = (int)(RING_BUDGET / W_BYTES);
// Ring stages fetched before the dependency wait in the fused-norm form. With
// the whole ring in flight, the loads of h after the wait queued behind those
// misses; measured on the LLaMA-7B layer's decode (per token): 11 stages
// 86.9 us, 8 86.1, 7 85.8, 6 85.8, 4 85.9. The plain form keeps its whole
// ring (its X tiles share the stages' barriers; 5 / 7 / 9 of 10 were slower).
constexpr int NORM_PREFETCH = 6;
// ring, resident rows, a 16-byte zero block (the MMA rows past M), the norm
// weight, output staging, barriers (ring + the weight's)
__host__ __device__ constexpr size_t gemv_norm_smem() {
  return 1024 + (size_t)NORM_STAGES * W_BYTES + (size_t)NORM_MAX_M * NORM_XS + 16 + (size_t)NORM_MAX_K * 2 +
         (size_t)8 * OS * 4 + 2 * NORM_STAGES * 8 + 8 + 16;
}
static_assert(gemv_norm_smem() <= 232448, "fused-norm GEMV shared memory");
}  // namespace

// swizzled byte address of (row, col) in a tile of 128-byte rows written by TMA
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int col) {
  return base + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4);
}

// Stream-K split: the row_blocks x nk weight stages (row block rb, k stage i
// -> index rb*nk + i) are cut into `grid` equal contiguous ranges, so every
// CTA streams the same number of bytes. CTA c owns [begin(c), begin(c+1)).
__host__ __device__ __forceinline__ int sk_begin(int c, int total, int grid) {
  return (int)(((long long)c * total) / grid);
}
// the CTA whose range holds stage x
__host__ __device__ __forceinline__ int sk_owner(int x, int total, int grid) {
  int c = (int)(((long long)x * grid) / total);
  while (c + 1 < grid && sk_begin(c + 1, total, grid) <= x) ++c;
  while (c > 0 && sk_begin(c, total, grid) > x) --c;
  return c;
}

// NORM (MB == 1, M <= NORM_MAX_M, K <= NORM_MAX_K): X = RMSNorm(h_norm) with
// weight w_norm and eps, computed here; map_x is not read.
template <int MB, bool NORM>
__global__ void __launch_bounds__(160, 1)
    llama_decode_linear_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x, int M,
                     int N, int nk, int total, int tiled, float* __restrict__ part, int* __restrict__ counters,
                     EpiParams ep, const float* __restrict__ h_norm, const bf16* __restrict__ w_norm, float eps) {
  static_assert(!NORM || MB == 1, "the fused norm serves one 8-token block");
  constexpr int STAGES = NORM ? NORM_STAGES : stages(MB);
  constexpr uint32_t SB = NORM ? W_BYTES : stage_bytes(MB);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xres = base + STAGES * SB;  // NORM: the M normalised rows, a zero block, the norm weight
  uint8_t* xzero = xres + NORM_MAX_M * NORM_XS;
  uint8_t* wsm = xzero + 16;
  float* os = reinterpret_cast<float*>(NORM ? wsm + NORM_MAX_K * 2 : xres);
  uint64_t* full = reinterpret_cast<uint64_t*>(os + 8 * MB * OS);
  uint64_t* empty = full + STAGES;
  uint64_t* wbar = empty + STAGES;  // NORM: the norm weight landed
  __shared__ int s_last;
  __shared__ int s_abort;
  __shared__ float s_ss[4][NORM_MAX_M];  // NORM: per-warp sums of squares of each row
  volatile int* abort_flag = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int grid = gridDim.x, cta = blockIdx.x;
  const int sbeg = sk_begin(cta, total, grid), send = sk_begin(cta + 1, total, grid);

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    if (NORM) mbar_init(wbar, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&map_w);
      prefetch_tensormap(&map_x);
      // The weights do not depend on the previous kernel: fill the ring with
      // weight tiles first, then wait for the producer of X and add X tiles.
      if constexpr (NORM) {
        mbar_arrive_expect_tx(wbar, (uint32_t)(nk * KB * 2));
        bulk_load(wsm, w_norm, (uint32_t)(nk * KB * 2), wbar);
      }
      const int pre = min(NORM ? NORM_PREFETCH : STAGES, send - sbeg);
      for (int i = 0; i < pre; ++i) {
        const int x = sbeg + i, rb = x / nk, ks = x - rb * nk;
        mbar_arrive_expect_tx(&full[i], SB);
        tma_load_2d(base + i * SB, &map_w, &full[i], tiled ? 0 : ks * KB, tiled ? (rb * nk + ks) * RPC : rb * RPC);
      }
      pdl_wait();
      pdl_trigger();
      if constexpr (!NORM) {
        for (int i = 0; i < pre; ++i) {
          const int x = sbeg + i, ks = x - (x / nk) * nk;
          tma_load_2d(base + i * SB + W_BYTES, &map_x, &full[i], ks * KB, 0);
        }
      }
      int j = pre;
      for (int x = sbeg + pre; x < send; ++x, ++j) {
        const int st = j % STAGES;
        if (!wait_or_abort(&empty[st], ((j / STAGES) & 1) ^ 1, ep.err, abort_flag)) break;
        const int rb = x / nk, ks = x - rb * nk;
        uint8_t* dst = base + st * SB;
        mbar_arrive_expect_tx(&full[st], SB);
        tma_load_2d(dst, &map_w, &full[st], tiled ? 0 : ks * KB, tiled ? (rb * nk + ks) * RPC : rb * RPC);
        if constexpr (!NORM) tma_load_2d(dst + W_BYTES, &map_x, &full[st], ks * KB, 0);
      }
      // the CTA must not retire while a copy into its shared memory is in flight
      for (int i = (j > STAGES ? j - STAGES : 0); i < j; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, ep.err);
      if constexpr (NORM) mbar_wait(wbar, 0, ep.err);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int K = nk * KB;
  pdl_wait();
  pdl_trigger();
  if constexpr (NORM) {
    // every load of this thread's share of the M rows is issued before any is used
    float4 hv[NORM_MAX_M][NORM_CHUNKS];
#pragma unroll
    for (int m = 0; m < NORM_MAX_M; ++m)
#pragma unroll
      for (int i = 0; i < NORM_CHUNKS; ++i) {
        const int c4 = (tid + 128 * i) * 4;
        hv[m][i] = (m < M && c4 < K) ? *reinterpret_cast<const float4*>(h_norm + (size_t)m * K + c4)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int m = 0; m < NORM_MAX_M; ++m) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < NORM_CHUNKS; ++i)
        ss += hv[m][i].x * hv[m][i].x + hv[m][i].y * hv[m][i].y + hv[m][i].z * hv[m][i].z + hv[m][i].w * hv[m][i].w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_ss[warp][m] = ss;
    }
    if (tid == 0) *reinterpret_cast<uint4*>(xzero) = make_uint4(0u, 0u, 0u, 0u);
    wait_or_abort(wbar, 0, ep.err, abort_flag);
    uint2 wn[NORM_CHUNKS];
#pragma unroll
    for (int i = 0; i < NORM_CHUNKS; ++i) {
      const int c4 = (tid + 128 * i) * 4;
      wn[i] = c4 < K ? *reinterpret_cast<const uint2*>(wsm + c4 * 2) : make_uint2(0u, 0u);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
    for (int m = 0; m < NORM_MAX_M; ++m) {
      if (m >= M) break;
      const float inv = rsqrtf((s_ss[0][m] + s_ss[1][m] + s_ss[2][m] + s_ss[3][m]) / (float)K + eps);
#pragma unroll
      for (int i = 0; i < NORM_CHUNKS; ++i) {
        const int c4 = (tid + 128 * i) * 4;
        if (c4 < K) {
          const float2 w0 = unpack_bf16x2(wn[i].x), w1 = unpack_bf16x2(wn[i].y);
          uint2 u;
          u.x = pack_bf16x2(round_to<bf16>(hv[m][i].x * inv) * w0.x, round_to<bf16>(hv[m][i].y * inv) * w0.y);
          u.y = pack_bf16x2(round_to<bf16>(hv[m][i].z * inv) * w1.x, round_to<bf16>(hv[m][i].w * inv) * w1.y);
          *reinterpret_cast<uint2*>(xres + m * NORM_XS + c4 * 2) = u;
        }
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  const int a_row = warp * 32 + (lane & 7) + 8 * ((lane >> 3) & 1);  // + 16 t
  const int a_col = 8 * (lane >> 4);                                 // + 16 kk
  int j = 0;
  int x = sbeg;
  while (x < send) {
    const int rb = x / nk;
    const int seg_beg = x, seg_end = min(send, (rb + 1) * nk);
    float acc[2][MB][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) acc[t][mb][0] = acc[t][mb][1] = acc[t][mb][2] = acc[t][mb][3] = 0.f;

    // On a timed-out wait the abort flag makes every later wait return at once:
    // the warps still walk the same stages and barriers, so the CTA unwinds
    // without a hang (results are then garbage, and the device flag says so).
    for (; x < seg_end; ++x, ++j) {
      const int st = j % STAGES;
      const bool ok = wait_or_abort(&full[st], (j / STAGES) & 1, ep.err, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        const uint32_t wb = smem_u32(base + st * SB);
        const uint32_t xb = wb + W_BYTES;
#pragma unroll
        for (int kk2 = 0; kk2 < 2; ++kk2) {
          uint32_t xf[MB][4];
          if constexpr (NORM) {
            // resident rows (plain row-major); rows past M read the zero block
            const int row = lane & 7, k0 = (x - rb * nk) * KB + kk2 * 32 + 8 * (lane >> 3);
            ldmatrix_x4(xf[0], row < M ? smem_u32(xres) + row * NORM_XS + k0 * 2 : smem_u32(xzero));
          } else {
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
              ldmatrix_x4(xf[mb], sw128(xb, mb * 8 + (lane & 7), kk2 * 32 + 8 * (lane >> 3)));
          }
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2) {
            const int kk = kk2 * 2 + s2;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              uint32_t a[4];
              ldmatrix_x4(a, sw128(wb, a_row + 16 * t, a_col + 16 * kk));
#pragma unroll
              for (int mb = 0; mb < MB; ++mb) {
                const uint32_t b[2] = {xf[mb][2 * s2], xf[mb][2 * s2 + 1]};
                mma_bf16_16816(acc[t][mb], a, b);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // fragment (row g / g+8 of each 16-row tile, tokens 2q, 2q+1 of each 8-token block) -> os[token][row]
    asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const int rl = warp * 32 + t * 16 + g;
        const int m = mb * 8 + 2 * q;
        os[m * OS + rl] = acc[t][mb][0];
        os[(m + 1) * OS + rl] = acc[t][mb][1];
        os[m * OS + rl + 8] = acc[t][mb][2];
        os[(m + 1) * OS + rl + 8] = acc[t][mb][3];
      }
    asm volatile("bar.sync 1, 128;" ::: "memory");

    const int nbase = rb * RPC;
    if (seg_beg == rb * nk && seg_end == (rb + 1) * nk) {
      // this CTA streamed the whole row block: epilogue straight from shared memory
      for (int c = tid; c < M * (RPC / 8); c += 128) {
        const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
        const int n = nbase + jc * 8;
        if (n < N) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = os[m * OS + jc * 8 + e];
          epilogue8<bf16>(ep, m, n, v);
        }
      }
      continue;
    }
    // partial row block: slot = this CTA's index among the row block's contributors
    const int c_first = sk_owner(rb * nk, total, grid);
    const int c_last = sk_owner((rb + 1) * nk - 1, total, grid);
    const int count = c_last - c_first + 1, slot = cta - c_first;
    for (int e = tid; e < M * (RPC / 4); e += 128) {
      const int m = e / (RPC / 4), jc = e - m * (RPC / 4);
      const int n = nbase + jc * 4;
      if (n < N) {
        const float4 v = make_float4(os[m * OS + jc * 4], os[m * OS + jc * 4 + 1], os[m * OS + jc * 4 + 2],
                                     os[m * OS + jc * 4 + 3]);
        __stcg(reinterpret_cast<float4*>(part + ((size_t)slot * M + m) * N + n), v);
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (tid == 0) s_last = (atomic_add_acq_rel(&counters[rb], 1) == count - 1);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!s_last) continue;
    for (int c = tid; c < M * (RPC / 8); c += 128) {
      const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
      const int n = nbase + jc * 8;
      if (n >= N) continue;
      // the residual row is fetched before the partial sums, not after them
      const bool res = ep.kind == EPI_RESIDUAL;
      float4* hp = res ? reinterpret_cast<float4*>(ep.out + (size_t)m * ep.ld_out + n) : nullptr;
      float4 h0 = make_float4(0.f, 0.f, 0.f, 0.f), h1 = h0;
      if (res) {
        h0 = hp[0];
        h1 = hp[1];
      }
      // the partials in slot order; the loads of up to 8 slots are issued before
      // any of them is added, so a chunk costs one L2 round trip, not one per slot
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int sl0 = 0; sl0 < count; sl0 += 8) {
        float4 pa[8], pb[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (sl0 + i < count) {
            const float4* src = reinterpret_cast<const float4*>(part + ((size_t)(sl0 + i) * M + m) * N + n);
            pa[i] = __ldcg(src);
            pb[i] = __ldcg(src + 1);
          }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (sl0 + i < count) {
            v[0] += pa[i].x; v[1] += pa[i].y; v[2] += pa[i].z; v[3] += pa[i].w;
            v[4] += pb[i].x; v[5] += pb[i].y; v[6] += pb[i].z; v[7] += pb[i].w;
          }
      }
      if (res) {
        hp[0] = make_float4(h0.x + v[0], h0.y + v[1], h0.z + v[2], h0.w + v[3]);
        hp[1] = make_float4(h1.x + v[4], h1.y + v[5], h1.z + v[6], h1.w + v[7]);
      } else {
        epilogue8<bf16>(ep, m, n, v);
      }
    }
    if (tid == 0) counters[rb] = 0;
  }
}

// tcgen05 form of the same kernel for 9..32 tokens (MB = 2 or 4; 17..24 tokens
// run as MB = 4, the X box's rows past M filled with zeros by the copy). The
// ring, the stream-K ranges, the partial workspace and the epilogue are those
// of llama_decode_linear_kernel; only the product changes: a sixth warp's
// elected thread issues tcgen05.mma with the stage's 128 weight rows as A
// (M = 128) and its 8 MB token rows as B (N = 8 MB), 4 MMAs of 16 k per stage,
// accumulating in tensor memory (two 32-column buffers, alternating between
// the row-block segments of the CTA's range), and frees the stage with a
// commit. The tensor core reads each stage once, where the warp-level form
// issues 32 mma.sync and 16 ldmatrix per warp and stage at 32 tokens (32 KB of
// shared-memory reads per 20 KB stage); measured, the two run at the same
// speed (see g_gemv_mma), so the warp-level form stays the default and this
// one is selected with llama_set_decode_linear_mma. The four epilogue warps read
// their 32 rows of the accumulator with tcgen05.ld (lane = weight row, column
// = token) into the same [token][row] staging tile.
template <int MB>
__global__ void __launch_bounds__(192, 1)
    llama_decode_linear_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                                  int M, int N, int nk, int total, int tiled, float* __restrict__ part,
                                  int* __restrict__ counters, EpiParams ep) {
  static_assert(MB == 2 || MB == 4, "N = 8 MB must be a multiple of 16 for M = 128");
  constexpr int STAGES = stages(MB);
  constexpr uint32_t SB = stage_bytes(MB);
  constexpr uint32_t IDESC = make_idesc_bf16(RPC, 8 * MB);
  constexpr uint32_t TMEM_COLS = 64;  // two accumulator buffers of 32 columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* os = reinterpret_cast<float*>(base + STAGES * SB);
  uint64_t* full = reinterpret_cast<uint64_t*>(os + 8 * MB * OS);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;  // [2] accumulator buffer complete
  uint64_t* aempty = afull + 2;      // [2] accumulator buffer read by the four epilogue warps
  uint64_t* drained = aempty + 2;    // every MMA of the CTA finished
  __shared__ uint32_t s_tmem;
  __shared__ int s_last;
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grid = gridDim.x, cta = blockIdx.x;
  const int sbeg = sk_begin(cta, total, grid), send = sk_begin(cta + 1, total, grid);

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&aempty[i], 4);
    }
    mbar_init(drained, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&map_w);
      prefetch_tensormap(&map_x);
      const int pre = min(STAGES, send - sbeg);
      for (int i = 0; i < pre; ++i) {
        const int x = sbeg + i, rb = x / nk, ks = x - rb * nk;
        mbar_arrive_expect_tx(&full[i], SB);
        tma_load_2d(base + i * SB, &map_w, &full[i], tiled ? 0 : ks * KB, tiled ? (rb * nk + ks) * RPC : rb * RPC);
      }
      pdl_wait();
      pdl_trigger();
      for (int i = 0; i < pre; ++i) {
        const int x = sbeg + i, ks = x - (x / nk) * nk;
        tma_load_2d(base + i * SB + W_BYTES, &map_x, &full[i], ks * KB, 0);
      }
      int j = pre;
      for (int x = sbeg + pre; x < send; ++x, ++j) {
        const int st = j % STAGES;
        if (!wait_or_abort(&empty[st], ((j / STAGES) & 1) ^ 1, ep.err, abort_flag)) break;
        const int rb = x / nk, ks = x - rb * nk;
        uint8_t* dst = base + st * SB;
        mbar_arrive_expect_tx(&full[st], SB);
        tma_load_2d(dst, &map_w, &full[st], tiled ? 0 : ks * KB, tiled ? (rb * nk + ks) * RPC : rb * RPC);
        tma_load_2d(dst + W_BYTES, &map_x, &full[st], ks * KB, 0);
      }
      // the CTA must not retire while a copy into its shared memory is in flight
      for (int i = (j > STAGES ? j - STAGES : 0); i < j; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, ep.err);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    pdl_trigger();
    if (lane == 0) {
      int j = 0, seg = 0;
      bool ok = true;
      for (int x = sbeg; x < send && ok; ++seg) {
        const int rb = x / nk, seg_end = min(send, (rb + 1) * nk);
        const int buf = seg & 1;
        if (!wait_or_abort(&aempty[buf], ((seg >> 1) & 1) ^ 1, ep.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * 32;
        for (bool first = true; x < seg_end; ++x, ++j, first = false) {
          const int st = j % STAGES;
          if (!wait_or_abort(&full[st], (j / STAGES) & 1, ep.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(base + st * SB), xa = wa + W_BYTES;
#pragma unroll
          for (int kk = 0; kk < KB / 16; ++kk)
            tc_mma_bf16(d, make_sw128_desc(wa + kk * 32), make_sw128_desc(xa + kk * 32), IDESC,
                        (first && kk == 0) ? 0u : 1u);
          tc_commit(&empty[st]);
        }
        if (ok) tc_commit(&afull[buf]);
      }
      // every MMA of this thread has finished before the tensor memory is released
      tc_commit(drained);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drained, 0) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
      }
    }
  } else {
    // ------------------------------------------------------- epilogue warps 0-3
    pdl_wait();
    pdl_trigger();
    const int row = warp * 32 + lane;  // weight row of the row block = TMEM lane
    int seg = 0;
    for (int x = sbeg; x < send; ++seg) {
      const int rb = x / nk;
      const int seg_beg = x, seg_end = min(send, (rb + 1) * nk);
      x = seg_end;
      const int buf = seg & 1;
      const bool ok = wait_or_abort(&afull[buf], (seg >> 1) & 1, ep.err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: tcgen05.ld is warp-collective
      tc_fence_after();
      float v[32];
      tmem_ld_32cols(tmem + ((uint32_t)(warp * 32) << 16) + buf * 32, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[buf]);

      asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
      for (int m = 0; m < 8 * MB; ++m) os[m * OS + row] = v[m];
      asm volatile("bar.sync 1, 128;" ::: "memory");

      const int nbase = rb * RPC;
      if (seg_beg == rb * nk && seg_end == (rb + 1) * nk) {
        for (int c = tid; c < M * (RPC / 8); c += 128) {
          const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
          const int n = nbase + jc * 8;
          if (n < N) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = os[m * OS + jc * 8 + e];
            epilogue8<bf16>(ep, m, n, o);
          }
        }
        continue;
      }
      const int c_first = sk_owner(rb * nk, total, grid);
      const int c_last = sk_owner((rb + 1) * nk - 1, total, grid);
      const int count = c_last - c_first + 1, slot = cta - c_first;
      for (int e = tid; e < M * (RPC / 4); e += 128) {
        const int m = e / (RPC / 4), jc = e - m * (RPC / 4);
        const int n = nbase + jc * 4;
        if (n < N) {
          const float4 o = make_float4(os[m * OS + jc * 4], os[m * OS + jc * 4 + 1], os[m * OS + jc * 4 + 2],
                                       os[m * OS + jc * 4 + 3]);
          __stcg(reinterpret_cast<float4*>(part + ((size_t)slot * M + m) * N + n), o);
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) s_last = (atomic_add_acq_rel(&counters[rb], 1) == count - 1);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!s_last) continue;
      for (int c = tid; c < M * (RPC / 8); c += 128) {
        const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
        const int n = nbase + jc * 8;
        if (n >= N) continue;
        const bool res = ep.kind == EPI_RESIDUAL;
        float4* hp = res ? reinterpret_cast<float4*>(ep.out + (size_t)m * ep.ld_out + n) : nullptr;
        float4 h0 = make_float4(0.f, 0.f, 0.f, 0.f), h1 = h0;
        if (res) {
          h0 = hp[0];
          h1 = hp[1];
        }
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int sl0 = 0; sl0 < count; sl0 += 8) {
          float4 pa[8], pb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (sl0 + i < count) {
              const float4* src = reinterpret_cast<const float4*>(part + ((size_t)(sl0 + i) * M + m) * N + n);
              pa[i] = __ldcg(src);
              pb[i] = __ldcg(src + 1);
            }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (sl0 + i < count) {
              o[0] += pa[i].x; o[1] += pa[i].y; o[2] += pa[i].z; o[3] += pa[i].w;
              o[4] += pb[i].x; o[5] += pb[i].y; o[6] += pb[i].z; o[7] += pb[i].w;
            }
        }
        if (res) {
          hp[0] = make_float4(h0.x + o[0], h0.y + o[1], h0.z + o[2], h0.w + o[3]);
          hp[1] = make_float4(h1.x + o[4], h1.y + o[5], h1.z + o[6], h1.w + o[7]);
        } else {
          epilogue8<bf16>(ep, m, n, o);
        }
      }
      if (tid == 0) counters[rb] = 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// grid = one CTA per SM (fewer if there are fewer stages than SMs); the
// partial workspace holds one [M][N] slice per contributor of the most-split
// row block.
//
// Where a whole number c >= 2 of CTAs per row block still keeps at least 85 %
// of the SMs streaming, the grid is row_blocks x c instead: every range then
// lies inside one row block (each CTA has one segment, one partial tile and at
// most one merge, and every row block exactly c contributors), rather than
// most CTAs straddling two row blocks. Measured on B200 (graphs of back-to-back
// launches, us): one token x [4096 x 4096] 10.7 -> 9.1 and [4096 x 11008]
// 17.9 -> 17.1; 16 tokens x [8192 x 8192] 25.5 -> 24.9; 32 tokens x [4096 x
// 4096] 15.5 -> 13.8 and [6144 x 4096] 17.1 -> 15.9; the 7B-layer decode step
// 85.9 -> 84.0 us per token.
GemvPlan plan_gemv(int M, int N, int K, int num_sms) {
  GemvPlan p;
  p.row_blocks = (N + RPC - 1) / RPC;
  p.nk = K / KB;
  p.total = p.row_blocks * p.nk;
  p.grid = p.total < num_sms ? p.total : num_sms;
  if (p.row_blocks <= num_sms) {
    const int c = num_sms / p.row_blocks;
    if (c >= 2 && p.row_blocks * c * 100 >= num_sms * 85 && p.nk >= c) p.grid = p.row_blocks * c;
  }
  int smax = 1;
  for (int rb = 0; rb < p.row_blocks; ++rb) {
    const int c = sk_owner((rb + 1) * p.nk - 1, p.total, p.grid) - sk_owner(rb * p.nk, p.total, p.grid) + 1;
    if (c > smax) smax = c;
  }
  p.S = smax;
  p.part_floats = smax > 1 ? (size_t)smax * M * N : 0;
  return p;
}

// Host-side walk of a plan with the kernel's own index functions: every
// weight stage belongs to exactly one CTA's range; a row block split across
// CTAs gets one partial slot per contributor, the slots are 0 .. count-1 with
// count <= S, and the partial workspace holds S x M x N floats.
bool check_gemv_plan(int M, int N, int K, int num_sms) {
  const GemvPlan p = plan_gemv(M, N, K, num_sms);
  if (p.grid < 1 || p.total < 1 || K % KB) return false;
  std::vector<int> seen(p.total, 0);
  std::vector<std::vector<int>> slots(p.row_blocks);
  std::vector<int> counts(p.row_blocks, -1);
  for (int cta = 0; cta < p.grid; ++cta) {
    const int sbeg = sk_begin(cta, p.total, p.grid), send = sk_begin(cta + 1, p.total, p.grid);
    if (sbeg >= send) return false;  // every CTA of the grid has work
    for (int x = sbeg; x < send;) {
      const int rb = x / p.nk, seg_beg = x, seg_end = std::min(send, (rb + 1) * p.nk);
      if (rb >= p.row_blocks) return false;
      for (int y = seg_beg; y < seg_end; ++y) ++seen[y];
      if (!(seg_beg == rb * p.nk && seg_end == (rb + 1) * p.nk)) {
        const int c_first = sk_owner(rb * p.nk, p.total, p.grid);
        const int c_last = sk_owner((rb + 1) * p.nk - 1, p.total, p.grid);
        const int count = c_last - c_first + 1, slot = cta - c_first;
        if (slot < 0 || slot >= count || count > p.S) return false;
        if (counts[rb] >= 0 && counts[rb] != count) return false;
        counts[rb] = count;
        slots[rb].push_back(slot);
      }
      x = seg_end;
    }
  }
  for (int v : seen)
    if (v != 1) return false;
  for (int rb = 0; rb < p.row_blocks; ++rb) {
    if (counts[rb] < 0) continue;
    std::vector<int> sl = slots[rb];
    std::sort(sl.begin(), sl.end());
    if ((int)sl.size() != counts[rb]) return false;
    for (int i = 0; i < counts[rb]; ++i)
      if (sl[i] != i) return false;
  }
  if (p.S > 1 && p.part_floats < (size_t)p.S * M * N) return false;
  return true;
}

template <int MB, bool NORM = false>
static cudaError_t launch_mb(const CUtensorMap& mw, const CUtensorMap& mx, int M, int N, const GemvPlan& p,
                             int tiled, float* part, int* counters, const EpiParams& ep, cudaStream_t st,
                             const float* h_norm = nullptr, const bf16* w_norm = nullptr, float eps = 0.f) {
  constexpr size_t smem = NORM ? gemv_norm_smem() : gemv_smem(MB);
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(llama_decode_linear_kernel<MB, NORM>, smem, attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(llama_decode_linear_kernel<MB, NORM>, dim3(p.grid), dim3(160), smem, st, mw, mx, M, N, p.nk,
                    p.total, tiled, part, counters, ep, h_norm, w_norm, eps);
}

template <int MB>
static cudaError_t launch_tc_mb(const CUtensorMap& mw, const CUtensorMap& mx, int M, int N, const GemvPlan& p,
                                int tiled, float* part, int* counters, const EpiParams& ep, cudaStream_t st) {
  constexpr size_t smem = gemv_smem(MB) + 64;
  static_assert(gemv_smem(MB) + 64 <= 232448, "tcgen05 decode GEMV shared memory");
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(llama_decode_linear_tc_kernel<MB>, smem, attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(llama_decode_linear_tc_kernel<MB>, dim3(p.grid), dim3(192), smem, st, mw, mx, M, N, p.nk,
                    p.total, tiled, part, counters, ep);
}

// Product of the batched (9..32-token) calls: LLAMA_GEMV_MMA_* (process-wide).
// AUTO takes the warp-level form: measured on B200 (CUDA graph of back-to-back
// launches, tiled weights, us per launch, warp-level against tcgen05): 32
// tokens x [28672 x 4096] 44.2 / 45.4, [4096 x 14336] 27.0 / 27.2, [6144 x
// 4096] 17.1 / 17.5, [4096 x 4096] 15.6 / 16.1; 16 tokens x [57344 x 8192]
// 148.2 / 150.8, [8192 x 28672] 75.5 / 76.1; 24 tokens x [6144 x 4096] 15.5 /
// 16.5. The product is not what bounds these calls (the 32-token weight
// stream runs at the same speed either way).
static std::atomic<int> g_gemv_mma{LLAMA_GEMV_MMA_AUTO};

int set_gemv_mma(int mode) {
  if (mode < LLAMA_GEMV_MMA_AUTO || mode > LLAMA_GEMV_MMA_TCGEN05) return -1;
  g_gemv_mma.store(mode, std::memory_order_relaxed);
  return 0;
}

bool gemv_can_fuse_norm(int M, int K) { return M >= 1 && M <= NORM_MAX_M && K % KB == 0 && K <= NORM_MAX_K; }

cudaError_t launch_gemv_bf16(const void* X, const void* W, int tiled, int M, int N, int K, const GemvPlan& p,
                             float* part, int* counters, const EpiParams& ep, int num_sms, cudaStream_t st,
                             const CUtensorMap* wmap, const float* h_norm, const void* w_norm, float eps) {
  (void)num_sms;
  const int MB = (M + 7) / 8;
  CUtensorMap mw, mx;
  if (wmap && tiled)
    mw = *wmap;  // the library's weights: encoded once when they were set
  else if (!make_tmap_weights(&mw, W, tiled, N, K, RPC))
    return cudaErrorInvalidValue;
  if (h_norm) {  // X = RMSNorm(h_norm), computed by the kernel
    // the weight is bulk-copied (16-byte aligned); h is read as float4
    if (!w_norm || !gemv_can_fuse_norm(M, K) || (reinterpret_cast<uintptr_t>(w_norm) & 15) ||
        (reinterpret_cast<uintptr_t>(h_norm) & 15))
      return cudaErrorInvalidValue;
    return launch_mb<1, true>(mw, mw, M, N, p, tiled, part, counters, ep, st, h_norm,
                              reinterpret_cast<const bf16*>(w_norm), eps);
  }
  if (MB >= 2 && g_gemv_mma.load(std::memory_order_relaxed) == LLAMA_GEMV_MMA_TCGEN05) {
    // 17..24 tokens take the 32-row box (rows past M read as zeros)
    const int mbt = MB == 2 ? 2 : 4;
    if (!make_tmap_bf16(&mx, X, M, K, 8 * mbt)) return cudaErrorInvalidValue;
    return mbt == 2 ? launch_tc_mb<2>(mw, mx, M, N, p, tiled, part, counters, ep, st)
                    : launch_tc_mb<4>(mw, mx, M, N, p, tiled, part, counters, ep, st);
  }
  if (!make_tmap_bf16(&mx, X, M, K, 8 * MB)) return cudaErrorInvalidValue;
  switch (MB) {
    case 1: return launch_mb<1>(mw, mx, M, N, p, tiled, part, counters, ep, st);
    case 2: return launch_mb<2>(mw, mx, M, N, p, tiled, part, counters, ep, st);
    case 3: return launch_mb<3>(mw, mx, M, N, p, tiled, part, counters, ep, st);
    default: return launch_mb<4>(mw, mx, M, N, p, tiled, part, counters, ep, st);
  }
}

}  // namespace llama
