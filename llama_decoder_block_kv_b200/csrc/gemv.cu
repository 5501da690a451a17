// Decode GEMM for a handful of tokens (M <= 32): C[M][N] = X[M][K] * W[N][K]^T.
//
// At decode time every weight byte is read once per step and the token count
// is tiny, so this kernel is bound by HBM bandwidth, not by tensor throughput
// (the KV-cache section of "LLaMa-1/2/3 原理+源码——拆解" makes the same
// point: with the cache the bottleneck becomes memory access).
//
// A CTA owns 128 weight rows and one slice of K. One producer warp streams the
// slice through a 6-stage shared-memory ring with TMA (128 rows x 64 bf16 per
// stage, 128-byte swizzle, no multicast); the CTA's slice of X is staged once
// in shared memory. Four consumer warps (32 weight rows each) run the
// warp-level bf16 tensor-core MMA with the weights as the 16-row operand
// ("swap AB"): one MMA covers 16 weight rows x 8 tokens x 16 k.
//
// When K is split, each CTA writes its fp32 partial tile to a workspace and
// bumps a per-row-block counter; the CTA that arrives last sums the slices in
// a fixed order (deterministic) and runs the epilogue, then re-zeroes the
// counter, so the workspace needs no clearing between launches.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int RPC = 128;        // weight rows per CTA
constexpr int KB = 64;          // k per ring stage (one 128-byte swizzle row)
constexpr int STAGES = 6;
constexpr uint32_t STAGE_BYTES = RPC * KB * 2;
constexpr int OS = RPC + 4;     // row stride of the fp32 output staging tile

__host__ __device__ constexpr int kc_max(int mb) { return mb <= 2 ? 512 : 1024; }
__host__ __device__ constexpr int xs_stride(int kc) { return kc + 8; }  // +16 B: ldmatrix rows hit distinct banks

__host__ __device__ constexpr size_t gemv_smem(int mb, int kc) {
  return 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)8 * mb * xs_stride(kc) * 2 + 2 * STAGES * 8 + 16;
}
}  // namespace

// swizzled byte address of (row, col) in a stage tile of 128-byte rows
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int col) {
  return base + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4);
}

template <int MB>
__global__ void __launch_bounds__(160)
    gemv_bf16_kernel(const __grid_constant__ CUtensorMap map_w, const bf16* __restrict__ X, int M, int N, int K,
                     int Kc, int S, float* __restrict__ part, int* __restrict__ counters, EpiParams ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  bf16* xs = reinterpret_cast<bf16*>(base + STAGES * STAGE_BYTES);
  const int XS = xs_stride(Kc);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xs) + (size_t)8 * MB * XS * 2);
  uint64_t* empty = full + STAGES;
  float* os = reinterpret_cast<float*>(xs);  // reused once the ring and xs are drained
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rb = blockIdx.x, split = blockIdx.y;
  const int kb = split * Kc, ke = min(K, kb + Kc);
  const int klen = ke - kb;
  const int nst = klen / KB;

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    fence_barrier_init();
  }
  // stage this CTA's slice of X (rows >= M are zero)
  const int cpr = klen / 8;
  for (int e = tid; e < 8 * MB * cpr; e += 160) {
    const int m = e / cpr, c = e - m * cpr;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < M) v = *reinterpret_cast<const uint4*>(X + (size_t)m * K + kb + c * 8);
    *reinterpret_cast<uint4*>(xs + m * XS + c * 8) = v;
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&map_w);
      int j = 0;
      for (; j < nst; ++j) {
        const int st = j % STAGES;
        if (!mbar_wait(&empty[st], ((j / STAGES) & 1) ^ 1, ep.err)) break;
        mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
        tma_load_2d(ring + st * STAGE_BYTES, &map_w, &full[st], kb + j * KB, rb * RPC);
      }
      for (int i = (j > STAGES ? j - STAGES : 0); i < j; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, ep.err);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  float acc[2][MB][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) acc[t][mb][0] = acc[t][mb][1] = acc[t][mb][2] = acc[t][mb][3] = 0.f;

  const uint32_t xs_base = smem_u32(xs);
  const int a_row = warp * 32 + (lane & 7) + 8 * ((lane >> 3) & 1);  // + 16 t
  const int a_col = 8 * (lane >> 4);                                 // + 16 kk
  for (int j = 0; j < nst; ++j) {
    const int st = j % STAGES;
    const bool ok = mbar_wait(&full[st], (j / STAGES) & 1, ep.err);
    if (!__all_sync(0xffffffffu, ok)) break;
    const uint32_t wb = smem_u32(ring + st * STAGE_BYTES);
#pragma unroll
    for (int kk2 = 0; kk2 < 2; ++kk2) {
      uint32_t xf[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
        ldmatrix_x4(xf[mb], xs_base + ((mb * 8 + (lane & 7)) * XS + j * KB + kk2 * 32 + 8 * (lane >> 3)) * 2);
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
  if (S == 1) {
    for (int c = tid; c < M * (RPC / 8); c += 128) {
      const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
      const int n = nbase + jc * 8;
      if (n < N) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = os[m * OS + jc * 8 + i];
        epilogue8<bf16>(ep, m, n, v);
      }
    }
    return;
  }

  for (int e = tid; e < M * (RPC / 4); e += 128) {
    const int m = e / (RPC / 4), jc = e - m * (RPC / 4);
    const int n = nbase + jc * 4;
    if (n < N) {
      const float4 v = make_float4(os[m * OS + jc * 4], os[m * OS + jc * 4 + 1], os[m * OS + jc * 4 + 2],
                                   os[m * OS + jc * 4 + 3]);
      __stcg(reinterpret_cast<float4*>(part + ((size_t)split * M + m) * N + n), v);
    }
  }
  __threadfence();
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (tid == 0) s_last = (atomicAdd(&counters[rb], 1) == S - 1);
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (!s_last) return;
  __threadfence();
  for (int c = tid; c < M * (RPC / 8); c += 128) {
    const int m = c / (RPC / 8), jc = c - m * (RPC / 8);
    const int n = nbase + jc * 8;
    if (n >= N) continue;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
      const float4* src = reinterpret_cast<const float4*>(part + ((size_t)s * M + m) * N + n);
      const float4 a = __ldcg(src), b = __ldcg(src + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    epilogue8<bf16>(ep, m, n, v);
  }
  if (tid == 0) counters[rb] = 0;
}

// The K split: slices of at most kc_max(MB) (the X staging buffer) and enough
// CTAs to keep every SM streaming (about 2 per SM).
GemvPlan plan_gemv(int M, int N, int K, int num_sms) {
  GemvPlan p;
  const int MB = (M + 7) / 8;
  p.row_blocks = (N + RPC - 1) / RPC;
  int S = (K + kc_max(MB) - 1) / kc_max(MB);
  const int want = (2 * num_sms + p.row_blocks - 1) / p.row_blocks;
  if (want > S) S = want;
  const int max_s = K / (2 * KB) > 0 ? K / (2 * KB) : 1;  // at least two stages per slice
  if (S > max_s) S = max_s;
  int Kc = (K + S - 1) / S;
  Kc = (Kc + KB - 1) / KB * KB;
  if (Kc > kc_max(MB)) Kc = kc_max(MB);
  p.Kc = Kc;
  p.S = (K + Kc - 1) / Kc;
  p.part_floats = p.S > 1 ? (size_t)p.S * M * N : 0;
  return p;
}

template <int MB>
static cudaError_t launch_mb(const CUtensorMap& map, const bf16* x, int M, int N, int K, const GemvPlan& p,
                             float* part, int* counters, const EpiParams& ep, cudaStream_t st) {
  const size_t smem = gemv_smem(MB, p.Kc);
  static size_t attr = 0;
  if (attr < smem) {
    cudaError_t e = cudaFuncSetAttribute(gemv_bf16_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemv_smem(MB, kc_max(MB)));
    if (e != cudaSuccess) return e;
    attr = gemv_smem(MB, kc_max(MB));
  }
  dim3 grid(p.row_blocks, p.S);
  gemv_bf16_kernel<MB><<<grid, 160, smem, st>>>(map, x, M, N, K, p.Kc, p.S, part, counters, ep);
  return cudaGetLastError();
}

cudaError_t launch_gemv_bf16(const void* X, const void* W, int M, int N, int K, const GemvPlan& p, float* part,
                             int* counters, const EpiParams& ep, cudaStream_t st) {
  CUtensorMap map;
  if (!make_tmap_bf16(&map, W, N, K, RPC)) return cudaErrorInvalidValue;
  const bf16* x = reinterpret_cast<const bf16*>(X);
  switch ((M + 7) / 8) {
    case 1: return launch_mb<1>(map, x, M, N, K, p, part, counters, ep, st);
    case 2: return launch_mb<2>(map, x, M, N, K, p, part, counters, ep, st);
    case 3: return launch_mb<3>(map, x, M, N, K, p, part, counters, ep, st);
    default: return launch_mb<4>(map, x, M, N, K, p, part, counters, ep, st);
  }
}

}  // namespace llama
