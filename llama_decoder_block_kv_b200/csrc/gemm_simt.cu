// fp32 CUDA-core GEMM, C[M][N] = A[M][K] * W[N][K]^T with fp32 FMA, handing
// each row's 8-column chunks to the shared epilogue. Used in fp32 mode, where
// tensor cores cannot give 1e-4 relative accuracy (tf32 keeps 10 mantissa bits).
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256;
}

template <typename T>
__global__ void __launch_bounds__(THREADS)
    gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W, int M, int N, int K, EpiParams ep) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int ty = tid / 8, tx = tid % 8;  // rows ty*2, ty*2+1; cols tx*8 .. tx*8+7
  float acc[2][8] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    // each thread stages 4 elements of A and 4 of W (64 x 16 tiles)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + i * THREADS;  // 0..1023
      const int r = e / BK, c = e % BK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? to_f32(A[(size_t)gm * K + gk]) : 0.f;
      Ws[c][r] = (gn < N && gk < K) ? to_f32(W[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float a0 = As[k][ty * 2], a1 = As[k][ty * 2 + 1];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float b = Ws[k][tx * 8 + j];
        acc[0][j] = fmaf(a0, b, acc[0][j]);
        acc[1][j] = fmaf(a1, b, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int m = m0 + ty * 2 + i, n = n0 + tx * 8;
    if (m < M && n < N) epilogue8<T>(ep, m, n, acc[i]);
  }
}

template <typename T>
void launch_gemm_simt(const void* A, const void* W, int M, int N, int K, const EpiParams& ep, cudaStream_t st) {
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  launch_pdl(gemm_simt_kernel<T>, grid, dim3(THREADS), 0, st, reinterpret_cast<const T*>(A),
             reinterpret_cast<const T*>(W), M, N, K, ep);
}

template void launch_gemm_simt<float>(const void*, const void*, int, int, int, const EpiParams&, cudaStream_t);
template void launch_gemm_simt<bf16>(const void*, const void*, int, int, int, const EpiParams&, cudaStream_t);

}  // namespace llama
