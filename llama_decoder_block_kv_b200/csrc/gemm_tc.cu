// Tensor-core GEMM for sm_100a: C[M][N] = A[M][K] * B[N][K]^T, bf16 operands,
// fp32 accumulation in tensor memory, fused epilogues.
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: 128-byte-swizzled A (128 x 64) and B (BN x 64)
//               tiles into a STAGES-deep shared-memory ring (full/empty mbarriers);
//   warp 1      allocates 2 x BN tensor-memory columns (two accumulators), and one
//               lane issues tcgen05.mma (M = 128, N = BN, K = 16 per instruction),
//               committing each ring slot back to the producer and each finished
//               accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes (one output row per
//               thread), the fused epilogue per 8-column chunk, then release the
//               accumulator so the next tile's MMAs overlap this tile's epilogue.
// Tiles are visited in groups of GROUP_M row blocks so that concurrently running
// CTAs share A and B panels in L2. All TMA loads are plain (no multicast).
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int BM = 128, BK = 64;
constexpr int GROUP_M = 16;
}  // namespace

template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr size_t SMEM = 1024 /*align slack*/ + (size_t)STAGES * (A_BYTES + B_BYTES) + 256 /*barriers*/;
};

struct TileCoord {
  int mb, nb;
};

__device__ __forceinline__ TileCoord tile_coord(int tile, int num_m, int num_n) {
  const int per_group = GROUP_M * num_n;
  const int group = tile / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(num_m - first_m, GROUP_M);
  const int local = tile - group * per_group;
  return {first_m + local % gm, local / gm};
}

template <typename T, int BN>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, int M, int N,
                   int K, int b_tiled, EpiParams ep) {
  using Cfg = TcCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * Cfg::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drained = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_k = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, num_m, num_n);
        for (int kb = 0; kb < num_k; ++kb, ++it) {
          const int stage = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait_or_abort(&empty[stage], ph ^ 1, ep.err, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::A_BYTES + Cfg::B_BYTES);
          tma_load_2d(sA + stage * Cfg::A_BYTES, &map_a, &full[stage], kb * BK, tc.mb * BM);
          if (b_tiled) {
            // B in 128-row x 64-k tiles, tile (rb, kb) at rows (rb * num_k + kb) * 128 of the map
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tma_load_2d(sB + stage * Cfg::B_BYTES + h * 16384, &map_b, &full[stage], 0,
                          ((tc.nb * (BN / 128) + h) * num_k + kb) * 128);
          } else {
            tma_load_2d(sB + stage * Cfg::B_BYTES, &map_b, &full[stage], kb * BK, tc.nb * BN);
          }
        }
      }
      if (!ok) {
        // let every issued copy land before the CTA can exit (bounded)
        const int first = it > STAGES ? it - STAGES : 0;
        for (int j = first; j < it; ++j) {
          uint64_t* bar = &full[j % STAGES];
          const uint32_t ph = (j / STAGES) & 1;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar, ph) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN);
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!wait_or_abort(&tempty[acc], aph ^ 1, ep.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        for (int kb = 0; kb < num_k; ++kb, ++it) {
          const int stage = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait_or_abort(&full[stage], ph, ep.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc_mma_bf16(d, make_sw128_desc(a_addr + kk * 32), make_sw128_desc(b_addr + kk * 32), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      // all MMAs issued by this thread have finished before TMEM is released
      tc_commit(drained);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drained, 0) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const TileCoord tc = tile_coord(tile, num_m, num_n);
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const bool ok = wait_or_abort(&tfull[acc], aph, ep.err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: tcgen05.ld is warp-collective
      tc_fence_after();
      const int m = tc.mb * BM + row;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld_32cols(tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN + c * 32, v);
        if (m < M) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = tc.nb * BN + c * 32 + j * 8;
            if (n < N) epilogue8<T>(ep, m, n, v + j * 8);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

// ---------------------------------------------------------------------------
// host side

// signature of the driver's cuTensorMapEncodeTiled (cuda.h), fetched at run
// time so the library needs no link against libcuda
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix with a box of
// 64 columns (128 bytes) by box_rows rows and 128-byte swizzling.
bool make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of a weight matrix [N][K]: row-major (box 64 columns x box_rows
// rows), or, when tiled, the library's tile layout [ceil(N/128)][K/64][128][64]
// seen as rows of 64 elements (box 64 x box_rows rows, one tile per 128 rows).
bool make_tmap_weights(CUtensorMap* map, const void* ptr, int tiled, uint64_t N, uint64_t K, uint32_t box_rows) {
  if (!tiled) return make_tmap_bf16(map, ptr, N, K, box_rows);
  const uint64_t rows = (N + 127) / 128 * 128 * (K / 64);
  return make_tmap_bf16(map, ptr, rows, 64, box_rows);
}

// 3-D bf16 tensor map over a row-major [d2][d1][d0] array with a box of
// b0 x b1 x b2 elements (b0 * 2 bytes = 128) and 128-byte swizzling.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                       uint32_t b1, uint32_t b2) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN>
static cudaError_t launch_tc(const void* A, const void* B, int b_tiled, int M, int N, int K, const EpiParams& ep,
                             int num_sms, cudaStream_t st, const CUtensorMap* bmap) {
  CUtensorMap ma, mb;
  if (!make_tmap_bf16(&ma, A, M, K, BM)) return cudaErrorInvalidValue;
  if (bmap && b_tiled)
    mb = *bmap;  // the library's weights: encoded once when they were set
  else if (!make_tmap_weights(&mb, B, b_tiled, N, K, b_tiled ? 128 : BN))
    return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(gemm_tc_kernel<bf16, BN>, TcCfg<BN>::SMEM, attr);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_pdl(gemm_tc_kernel<bf16, BN>, dim3(grid), dim3(192), TcCfg<BN>::SMEM, st, ma, mb, M, N, K, b_tiled,
                    ep);
}

// BN = 256 unless that leaves the last wave badly filled.
cudaError_t launch_gemm_tc(const void* A, const void* B, int b_tiled, int M, int N, int K, const EpiParams& ep,
                           int num_sms, cudaStream_t st, const CUtensorMap* bmap) {
  const int num_m = (M + BM - 1) / BM;
  const int t256 = num_m * ((N + 255) / 256);
  const int t128 = num_m * ((N + 127) / 128);
  auto eff = [&](int tiles, double cost) {
    const int waves = (tiles + num_sms - 1) / num_sms;
    return (double)waves * cost;  // time ~ waves x per-tile cost
  };
  const bool use256 = (N % 256 == 0) && eff(t256, 2.0) <= eff(t128, 1.0) * 1.05;
  return use256 ? launch_tc<256>(A, B, b_tiled, M, N, K, ep, num_sms, st, bmap)
                : launch_tc<128>(A, B, b_tiled, M, N, K, ep, num_sms, st, bmap);
}

}  // namespace llama
