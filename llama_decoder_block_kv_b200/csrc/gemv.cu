// Decode GEMM for a handful of tokens (M <= 32): C[M][N] = X[M][K] * W[N][K]^T.
//
// At decode time every weight byte is read once per step and the token count
// is tiny, so this kernel is bound by HBM bandwidth, not by tensor throughput
// (the KV-cache section of "LLaMa-1/2/3 原理+源码——拆解" makes the same
// point: with the cache the bottleneck becomes memory access). The weights
// stream straight from HBM with 16-byte non-L1-allocating loads, several per
// thread in flight; the activations of the CTA's K slice are staged once in
// shared memory; the products run on the warp-level tensor-core MMA with the
// weights as the 16-row operand ("swap AB"), so one MMA covers 16 weight rows
// times 8 tokens.
//
// Work split: a CTA owns 128 weight rows (4 warps x 32) and one slice of K.
// When K is split, each CTA writes its fp32 partial tile to a workspace and
// bumps a per-row-block counter; the CTA that arrives last sums the slices in
// a fixed order (deterministic) and runs the epilogue, then re-zeroes the
// counter, so the workspace needs no clearing between launches.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int ROWS_PER_CTA = 128;
constexpr int KS = 512;        // K elements of X staged per shared-memory pass
constexpr int XS = KS + 32;    // padded row (64 B pad: rows alternate bank halves)
constexpr int OS = ROWS_PER_CTA + 4;
}  // namespace

// The 32 K-values a thread group touches per step are assigned to the MMA's
// logical k positions in a permuted but consistent order (the contraction is
// order-free): thread (g, q) loads physical k 8q..8q+7 of its rows as one
// 16-byte vector; physical pairs {0,1},{2,3} feed MMA step 0 (logical 2q and
// 2q+8), pairs {4,5},{6,7} feed step 1. The same map is applied to X.
template <int MB>
__device__ __forceinline__ void gemv_k32(float (&acc)[2][MB][4], const uint4 (&wv)[4], const bf16* xs, int kx, int g,
                                         int q) {
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    const uint4 xv = *reinterpret_cast<const uint4*>(xs + (mb * 8 + g) * XS + kx + 8 * q);
    const uint32_t b0[2] = {xv.x, xv.y};
    const uint32_t b1[2] = {xv.z, xv.w};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t a0[4] = {wv[2 * t].x, wv[2 * t + 1].x, wv[2 * t].y, wv[2 * t + 1].y};
      const uint32_t a1[4] = {wv[2 * t].z, wv[2 * t + 1].z, wv[2 * t].w, wv[2 * t + 1].w};
      mma_bf16_16816(acc[t][mb], a0, b0);
      mma_bf16_16816(acc[t][mb], a1, b1);
    }
  }
}

template <int MB>
__global__ void __launch_bounds__(128) gemv_bf16_kernel(const bf16* __restrict__ X, const bf16* __restrict__ W, int M,
                                                        int N, int K, int Kc, int S, float* __restrict__ part,
                                                        int* __restrict__ counters, EpiParams ep) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* xs = reinterpret_cast<bf16*>(smem_raw);       // [8*MB][XS]
  float* os = reinterpret_cast<float*>(smem_raw);     // [8*MB][OS], reused after the main loop
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rb = blockIdx.x, split = blockIdx.y;
  const int row0 = rb * ROWS_PER_CTA + warp * 32;
  const int kb = split * Kc, ke = min(K, kb + Kc);

  // rows of the 4 fragments: tile 0 rows g and g+8, tile 1 rows 16+g and 24+g
  const bf16* wr[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = row0 + (i >> 1) * 16 + (i & 1) * 8 + g;
    r = min(r, N - 1);
    wr[i] = W + (size_t)r * K + 8 * q;
  }

  float acc[2][MB][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][mb][j] = 0.f;

  for (int k0 = kb; k0 < ke; k0 += KS) {
    const int klen = min(KS, ke - k0);
    const int cpr = klen / 8;  // 16-byte chunks per row
    __syncthreads();
    for (int e = tid; e < 8 * MB * cpr; e += 128) {
      const int m = e / cpr, c = e - m * cpr;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (m < M) v = *reinterpret_cast<const uint4*>(X + (size_t)m * K + k0 + c * 8);
      *reinterpret_cast<uint4*>(xs + m * XS + c * 8) = v;
    }
    __syncthreads();
    int kk = 0;
    for (; kk + 128 <= klen; kk += 128) {
      uint4 wv[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) wv[u][i] = ldg_stream(wr[i] + k0 + kk + u * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u) gemv_k32<MB>(acc, wv[u], xs, kk + u * 32, g, q);
    }
    for (; kk < klen; kk += 32) {
      uint4 wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wv[i] = ldg_stream(wr[i] + k0 + kk);
      gemv_k32<MB>(acc, wv, xs, kk, g, q);
    }
  }

  // fragment (row g / g+8, tokens 2q, 2q+1 of each 8-token block) -> os[token][row]
  __syncthreads();
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
  __syncthreads();

  const int nbase = rb * ROWS_PER_CTA;
  if (S == 1) {
    for (int c = tid; c < M * (ROWS_PER_CTA / 8); c += 128) {
      const int m = c / (ROWS_PER_CTA / 8), j = c - m * (ROWS_PER_CTA / 8);
      const int n = nbase + j * 8;
      if (n < N) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = os[m * OS + j * 8 + i];
        epilogue8<bf16>(ep, m, n, v);
      }
    }
    return;
  }

  for (int e = tid; e < M * (ROWS_PER_CTA / 4); e += 128) {
    const int m = e / (ROWS_PER_CTA / 4), j = e - m * (ROWS_PER_CTA / 4);
    const int n = nbase + j * 4;
    if (n < N) {
      const float4 v = make_float4(os[m * OS + j * 4], os[m * OS + j * 4 + 1], os[m * OS + j * 4 + 2],
                                   os[m * OS + j * 4 + 3]);
      __stcg(reinterpret_cast<float4*>(part + ((size_t)split * M + m) * N + n), v);
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counters[rb], 1) == S - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int c = tid; c < M * (ROWS_PER_CTA / 8); c += 128) {
    const int m = c / (ROWS_PER_CTA / 8), j = c - m * (ROWS_PER_CTA / 8);
    const int n = nbase + j * 8;
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

// Chooses the K split so that the grid covers the SMs about twice.
GemvPlan plan_gemv(int M, int N, int K, int num_sms) {
  GemvPlan p;
  p.row_blocks = (N + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  int S = (2 * num_sms + p.row_blocks - 1) / p.row_blocks;
  const int max_s = K / 256 > 0 ? K / 256 : 1;
  if (S > max_s) S = max_s;
  if (S < 1) S = 1;
  int Kc = (K + S - 1) / S;
  Kc = (Kc + 63) / 64 * 64;
  p.Kc = Kc;
  p.S = (K + Kc - 1) / Kc;
  p.part_floats = p.S > 1 ? (size_t)p.S * M * N : 0;
  return p;
}

void launch_gemv_bf16(const void* X, const void* W, int M, int N, int K, const GemvPlan& p, float* part,
                      int* counters, const EpiParams& ep, cudaStream_t st) {
  const int MB = (M + 7) / 8;
  dim3 grid(p.row_blocks, p.S);
  const size_t xs_bytes = (size_t)8 * MB * XS * sizeof(bf16);
  const size_t os_bytes = (size_t)8 * MB * OS * sizeof(float);
  const size_t smem = xs_bytes > os_bytes ? xs_bytes : os_bytes;
  const bf16* x = reinterpret_cast<const bf16*>(X);
  const bf16* w = reinterpret_cast<const bf16*>(W);
  switch (MB) {
    case 1: gemv_bf16_kernel<1><<<grid, 128, smem, st>>>(x, w, M, N, K, p.Kc, p.S, part, counters, ep); break;
    case 2: gemv_bf16_kernel<2><<<grid, 128, smem, st>>>(x, w, M, N, K, p.Kc, p.S, part, counters, ep); break;
    case 3: gemv_bf16_kernel<3><<<grid, 128, smem, st>>>(x, w, M, N, K, p.Kc, p.S, part, counters, ep); break;
    default: gemv_bf16_kernel<4><<<grid, 128, smem, st>>>(x, w, M, N, K, p.Kc, p.S, part, counters, ep); break;
  }
}

}  // namespace llama
