// fp32 CUDA-core GEMM, C[M][N] = A[M][K] * W[N][K]^T with fp32 FMA, handing
// each row's 8-column chunks to the shared epilogue. Used in fp32 mode, where
// tensor cores cannot give 1e-4 relative accuracy (tf32 keeps 10 mantissa bits).
//
// A 64 x 64 output tile per CTA of 256 threads; K advances in steps of 16
// through a 4-stage shared-memory ring (40 KB for fp32) filled with 16-byte
// cp.async copies (zero-filled past the matrix edges), so the global-load
// latency of one step overlaps the FMAs of the three before it. Thread (ty, tx) accumulates rows
// 2ty, 2ty + 1 and columns tx + 8j (j < 8), which keeps the shared-memory reads
// of a warp on distinct banks; the tile then passes through shared memory so
// that each thread hands 8 consecutive columns of one row to the epilogue.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256, STAGES = 4;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  const uint32_t bytes = valid ? 16u : 0u;  // 0: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T>
struct SimtCfg {
  static constexpr int CE = 16 / sizeof(T);   // elements per 16-byte copy
  static constexpr int LDS = BK + CE;         // padded row stride (elements), a multiple of 16 bytes
  static constexpr int TILE = BM * LDS;       // elements of one A (or W) stage
};

template <typename T>
__global__ void __launch_bounds__(THREADS)
    gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W, int M, int N, int K, EpiParams ep) {
  using Cfg = SimtCfg<T>;
  extern __shared__ __align__(16) uint8_t simt_smem[];
  T* As = reinterpret_cast<T*>(simt_smem);            // [STAGES][BM][LDS]
  T* Ws = As + STAGES * Cfg::TILE;                      // [STAGES][BN][LDS]
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int ty = tid >> 3, tx = tid & 7;
  const int nk = (K + BK - 1) / BK;

  pdl_wait();
  pdl_trigger();

  // stage `st` <- k step `kb`: BM rows x BK elements of A and of W, CE per copy
  auto load = [&](int st, int kb) {
    constexpr int per_row = BK / Cfg::CE;
    for (int e = tid; e < BM * per_row; e += THREADS) {
      const int r = e / per_row, c = (e - r * per_row) * Cfg::CE;
      const int gk = kb * BK + c;
      const bool ka = gk < K;  // K % CE == 0, so a copy is wholly in or out
      const int gm = m0 + r, gn = n0 + r;
      cp_async16(As + st * Cfg::TILE + r * Cfg::LDS + c, A + (size_t)(gm < M ? gm : 0) * K + (ka ? gk : 0),
                 ka && gm < M);
      cp_async16(Ws + st * Cfg::TILE + r * Cfg::LDS + c, W + (size_t)(gn < N ? gn : 0) * K + (ka ? gk : 0),
                 ka && gn < N);
    }
  };

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nk) load(s, s);
    cp_async_commit();
  }
  float acc[2][8] = {};
  for (int kb = 0; kb < nk; ++kb) {
    cp_async_wait<STAGES - 2>();  // step kb has landed (the groups after it may still be in flight)
    __syncthreads();              // ... for every thread; and stage (kb - 1) % STAGES is free again
    if (kb + STAGES - 1 < nk) load((kb + STAGES - 1) % STAGES, kb + STAGES - 1);
    cp_async_commit();
    const T* as = As + (kb % STAGES) * Cfg::TILE;
    const T* ws = Ws + (kb % STAGES) * Cfg::TILE;
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float a0 = to_f32(as[(2 * ty) * Cfg::LDS + k]), a1 = to_f32(as[(2 * ty + 1) * Cfg::LDS + k]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float b = to_f32(ws[(tx + 8 * j) * Cfg::LDS + k]);
        acc[0][j] = fmaf(a0, b, acc[0][j]);
        acc[1][j] = fmaf(a1, b, acc[1][j]);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  // the 64 x 64 tile through shared memory: thread t then owns row t / 4, columns 16 (t % 4) .. + 15
  float* Cs = reinterpret_cast<float*>(simt_smem);  // [BM][BN + 4]
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) Cs[(2 * ty + i) * (BN + 4) + tx + 8 * j] = acc[i][j];
  __syncthreads();
  const int r = tid >> 2, c0 = (tid & 3) * 16;
  const int m = m0 + r;
  if (m < M) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + c0 + 8 * h;
      if (n < N) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = Cs[r * (BN + 4) + c0 + 8 * h + e];
        epilogue8<T>(ep, m, n, v);
      }
    }
  }
}

template <typename T>
size_t simt_smem_bytes() {
  const size_t ring = (size_t)2 * STAGES * SimtCfg<T>::TILE * sizeof(T);
  const size_t ctile = (size_t)BM * (BN + 4) * sizeof(float);
  return ring > ctile ? ring : ctile;
}

// fp32 decode GEMV for a few tokens (M <= 8, K <= 1024, K % 4 == 0, N % 8 ==
// 0): in the tiled kernel above a call of one token fills one row of a 64-row
// tile and walks K in 16-wide steps, one dependent round trip per ring stage,
// so a decode step of a small fp32 model is a chain of latencies. Here a CTA
// of 8 warps computes 8 consecutive output columns for all M tokens, warp w
// column n0 + w: each lane loads its K / 128 float4 of that weight row before
// the dependency wait (the weights do not depend on the previous kernel), the
// token rows are staged in shared memory after it, each sum is a warp
// reduction, and M threads hand the 8 columns of their token to the shared
// epilogue.
namespace {
constexpr int GV_KMAX = 1024, GV_MMAX = 8;
}

__global__ void __launch_bounds__(256)
    llama_decode_linear_f32_kernel(const float* __restrict__ A, const float* __restrict__ W, int M, int N, int K, EpiParams ep) {
  __shared__ float4 xs[GV_MMAX * GV_KMAX / 4];  // the M token rows, GV_KMAX floats apart
  __shared__ float res[GV_MMAX][8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * 8, n = n0 + warp;
  const int K4 = K >> 2;
  float4 wv[GV_KMAX / 128];
#pragma unroll
  for (int i = 0; i < GV_KMAX / 128; ++i) {
    const int k4 = lane + 32 * i;
    wv[i] = (n < N && k4 < K4) ? __ldg(reinterpret_cast<const float4*>(W + (size_t)n * K) + k4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  pdl_wait();
  for (int i = tid; i < M * K4; i += 256) {
    const int m = i / K4;
    xs[m * (GV_KMAX / 4) + (i - m * K4)] = reinterpret_cast<const float4*>(A)[i];
  }
  __syncthreads();
  pdl_trigger();
#pragma unroll
  for (int m = 0; m < GV_MMAX; ++m) {
    if (m >= M) break;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < GV_KMAX / 128; ++i) {
      const int k4 = lane + 32 * i;
      if (k4 < K4) {
        const float4 x = xs[m * (GV_KMAX / 4) + k4];
        acc = fmaf(wv[i].x, x.x, acc);
        acc = fmaf(wv[i].y, x.y, acc);
        acc = fmaf(wv[i].z, x.z, acc);
        acc = fmaf(wv[i].w, x.w, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) res[m][warp] = acc;
  }
  __syncthreads();
  if (tid < M) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = res[tid][e];
    epilogue8<float>(ep, tid, n0, v);
  }
}

template <typename T>
void launch_gemm_simt(const void* A, const void* W, int M, int N, int K, const EpiParams& ep, cudaStream_t st) {
  if constexpr (sizeof(T) == 4) {
    if (M >= 1 && M <= GV_MMAX && K <= GV_KMAX && K % 4 == 0 && N % 8 == 0 &&
        !(reinterpret_cast<uintptr_t>(A) & 15) && !(reinterpret_cast<uintptr_t>(W) & 15)) {
      launch_pdl(llama_decode_linear_f32_kernel, dim3(N / 8), dim3(256), 0, st, reinterpret_cast<const float*>(A),
                 reinterpret_cast<const float*>(W), M, N, K, ep);
      return;
    }
  }
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  launch_pdl(gemm_simt_kernel<T>, grid, dim3(THREADS), simt_smem_bytes<T>(), st, reinterpret_cast<const T*>(A),
             reinterpret_cast<const T*>(W), M, N, K, ep);
}

template void launch_gemm_simt<float>(const void*, const void*, int, int, int, const EpiParams&, cudaStream_t);
template void launch_gemm_simt<bf16>(const void*, const void*, int, int, int, const EpiParams&, cudaStream_t);

}  // namespace llama
