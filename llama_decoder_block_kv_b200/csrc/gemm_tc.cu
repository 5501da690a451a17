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
// The 2-SM form: a CTA pair (cluster of two) computes 256 x 256 tiles of C with
// tcgen05.mma.cta_group::2 (M = 256). Each CTA loads its 128 rows of A and one
// 128-row block of B (the library's tile layout: blocks 2 nb and 2 nb + 1 of
// the tile's 256 columns) into its own ring; the copies of both complete on
// rank 0's ring barriers (primed with both CTAs' bytes). Rank 0, warp 1, lane 0
// issues every MMA; ring slots and accumulators are released by commits that
// arrive on both CTAs' barriers. Each CTA's epilogue reads its own 128 rows
// from its TMEM; the accumulator goes back to the issuer once the epilogue
// threads of both CTAs have arrived on rank 0's barrier (rank 1's remotely).
// On B200 a 2-SM MMA with N = 256 costs ~134 cycles against ~168 for the 1-SM
// form with A in shared memory (measured), and each SM reads half of B.
namespace {
constexpr int P_BN = 256;
constexpr int P_STAGES = 6;
constexpr uint32_t P_A_BYTES = BM * BK * 2;        // this CTA's 128 rows of A
constexpr uint32_t P_B_BYTES = 128 * BK * 2;       // this CTA's 128 rows of B
constexpr size_t P_SMEM = 1024 + (size_t)P_STAGES * (P_A_BYTES + P_B_BYTES) + 256;
}  // namespace

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, int M,
                        int N, int K, EpiParams ep, int splits, float* __restrict__ ws, int* __restrict__ sync) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + P_STAGES * P_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + P_STAGES * P_B_BYTES);  // [P_STAGES] rank 0's: both CTAs' copies
  uint64_t* empty = full + P_STAGES;                                          // [P_STAGES] ring slot consumed
  uint64_t* tfull = empty + P_STAGES;   // [2] accumulator complete
  uint64_t* tempty = tfull + 2;         // [2] rank 0's: both CTAs' epilogues have read it
  uint64_t* drained = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_m = (M + 255) / 256, num_n = (N + P_BN - 1) / P_BN;
  const int num_tiles = num_m * num_n;
  const int num_k = (K + BK - 1) / BK;
  const int units = num_tiles * splits;  // (tile, k half) work units, the halves of a tile adjacent

  if (threadIdx.x == 0) {
    for (int i = 0; i < P_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * 128);
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
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(2 * P_BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any copy or commit reaches them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int it = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs) {
        const int tile = u / splits, s = u - tile * splits;
        const TileCoord tc = tile_coord(tile, num_m, num_n);
        for (int kb = s * num_k / splits; kb < (s + 1) * num_k / splits; ++kb, ++it) {
          const int stage = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (!wait_or_abort(&empty[stage], ph ^ 1, ep.err, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (P_A_BYTES + P_B_BYTES));
          const uint32_t bar = mbar_cluster_addr(&full[stage], 0);
          tma_load_2d_pair(sA + stage * P_A_BYTES, &map_a, bar, kb * BK, tc.mb * 256 + (int)rank * 128);
          // B in 128-row x 64-k tiles, tile (rb, kb) at rows (rb * num_k + kb) * 128 of the map
          tma_load_2d_pair(sB + stage * P_B_BYTES, &map_b, bar, 0, ((tc.nb * 2 + (int)rank) * num_k + kb) * 128);
        }
      }
      if (rank == 0) {
        // every copy of either CTA lands before the pair can retire (bounded): rank
        // 0's barriers count both CTAs' bytes, and rank 1 does not pass the final
        // cluster barrier before rank 0 has waited for them
        const int first = it > P_STAGES ? it - P_STAGES : 0;
        for (int j = first; j < it; ++j) {
          uint64_t* bar = &full[j % P_STAGES];
          const uint32_t ph = (j / P_STAGES) & 1;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar, ph) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (rank 0)
      constexpr uint32_t idesc = idesc2_bf16(256, P_BN, false);
      int it = 0, local = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs, ++local) {
        const int s = u % splits;
        const int kb0 = s * num_k / splits, kb1 = (s + 1) * num_k / splits;
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!wait_cluster_or_abort(&tempty[acc], aph ^ 1, ep.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * P_BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int stage = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (!wait_or_abort(&full[stage], ph, ep.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * P_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * P_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma2_ss(d, make_sw128_desc(a_addr + kk * 32), make_sw128_desc(b_addr + kk * 32), idesc,
                    (kb != kb0 || kk != 0) ? 1u : 0u);
          commit2(&empty[stage]);
        }
        if (!ok) break;
        commit2(&tfull[acc]);
      }
      // all MMAs have finished before TMEM is released
      commit2(drained);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drained, 0) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int local = 0;
    for (int u = pair; u < units; u += npairs, ++local) {
      const int tile = u / splits;
      const TileCoord tc = tile_coord(tile, num_m, num_n);
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const bool ok = wait_or_abort(&tfull[acc], aph, ep.err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: tcgen05.ld is warp-collective
      tc_fence_after();
      const int m = tc.mb * 256 + (int)rank * 128 + row;
      const uint32_t tacc = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * P_BN;
      // Split tiles: the warp's 32 rows of the two k halves meet here. The
      // first half to finish stores its sums ([column][row], 32 KB per warp)
      // and raises a flag; the second adds them to its own and runs the
      // epilogue (p0 + p1 = p1 + p0 in fp32, so the bits do not depend on
      // which finished first), then re-arms the counter and the flag.
      bool first = false, merge = false;
      float* wp = nullptr;
      int* cnt = nullptr;
      if (splits > 1) {
        const int slot = (tile * 2 + (int)rank) * 4 + quarter;
        cnt = sync + 2 * slot;
        wp = ws + (size_t)slot * (P_BN * 32);
        int f = 0;
        if (lane == 0) f = atomic_add_acq_rel(cnt, 1) == 0;
        first = __shfl_sync(0xffffffffu, f, 0) != 0;
        if (!first) {
          int got = 1;
          if (lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (!(got = ld_acquire_gpu(cnt + 1)) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
            }
            if (!got) atomicOr(ep.err, LLAMA_DEV_TIMEOUT);
          }
          merge = __shfl_sync(0xffffffffu, got, 0) != 0;
          __syncwarp();  // orders the other lanes' loads of the partial sums after lane 0's acquire
        }
      }
#pragma unroll 1
      for (int c = 0; c < P_BN / 32; ++c) {
        float v[32];
        tmem_ld_32cols(tacc + c * 32, v);
        if (first) {
#pragma unroll
          for (int j = 0; j < 32; ++j) __stcg(wp + (c * 32 + j) * 32 + lane, v[j]);
          continue;
        }
        if (merge) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += __ldcg(wp + (c * 32 + j) * 32 + lane);
        }
        if (m < M) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = tc.nb * P_BN + c * 32 + j * 8;
            if (n < N) epilogue8<T>(ep, m, n, v + j * 8);
          }
        }
      }
      if (first) {
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          st_release_gpu(cnt + 1, 1);
        }
      } else if (splits > 1 && lane == 0) {
        cnt[0] = 0;
        cnt[1] = 0;
      }
      tc_fence_before();
      // the reads above have completed (tcgen05.ld waits), so rank 1's arrival can be relaxed
      if (rank == 0) mbar_arrive(&tempty[acc]);
      else mbar_arrive_remote_relaxed(&tempty[acc], 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  // the other CTA's shared memory and TMEM are used by the pair's MMAs until
  // `drained`; neither CTA frees its TMEM or retires before both get here
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * P_BN) : "memory");
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

// CTA pairs over 256 x 256 tiles; B is the library's tiled weights (its map, 128-row boxes)
static cudaError_t launch_tc_pair(const void* A, const CUtensorMap& mb, int M, int N, int K, const EpiParams& ep,
                                  int num_sms, cudaStream_t st, int splits, float* ws, int* sync) {
  CUtensorMap ma;
  if (!make_tmap_bf16(&ma, A, M, K, BM)) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(gemm_tc_pair_kernel<bf16>, P_SMEM, attr);
  if (e != cudaSuccess) return e;
  const int units = ((M + 255) / 256) * ((N + P_BN - 1) / P_BN) * splits;
  const int pairs = units < num_sms / 2 ? units : num_sms / 2;
  return launch_pdl(gemm_tc_pair_kernel<bf16>, dim3(2 * pairs), dim3(192), P_SMEM, st, ma, mb, M, N, K, ep, splits,
                    ws, sync);
}

size_t gemm_split_ws_floats(int tiles) { return (size_t)tiles * 2 * 128 * P_BN; }
size_t gemm_split_sync_ints(int tiles) { return (size_t)tiles * 2 * 4 * 2; }
int gemm_split_max_tiles(int num_sms) { return 3 * (num_sms / 2); }

// The tile shape with the smallest estimate of waves x tile time, in units of a
// 1-SM 128 x 256 tile: 1-SM 128 x 128 tiles 0.5, 128 x 256 tiles 1, CTA-pair
// 256 x 256 tiles 0.7 (two SMs; the MMA step alone is ~134 against ~168 cycles,
// and whole GEMMs measured 0.69-0.75 of the single-CTA time); the pair form for
// weights in the library's tile layout only.
cudaError_t launch_gemm_tc(const void* A, const void* B, int b_tiled, int M, int N, int K, const EpiParams& ep,
                           int num_sms, cudaStream_t st, const CUtensorMap* bmap, const GemmSplitWs* split) {
  const int num_m = (M + BM - 1) / BM;
  const int t256 = num_m * ((N + 255) / 256);
  const int t128 = num_m * ((N + 127) / 128);
  const int tpair = ((M + 255) / 256) * ((N + 255) / 256);
  auto eff = [](int tiles, int slots, double cost) {
    const int waves = (tiles + slots - 1) / slots;
    return (double)waves * cost;  // time ~ waves x per-tile cost
  };
  const double e128 = eff(t128, num_sms, 0.5), e256 = eff(t256, num_sms, 1.0);
  double epair = eff(tpair, num_sms / 2, 0.7);
  // Two k halves per pair tile (run on different pairs; the second to finish
  // adds the first's partial sums) where that fills pairs a single wave of
  // whole tiles leaves idle. A half costs 0.35 plus 12 / num_k for the
  // partial tile's round trip through L2 and the unit's fixed cost, fitted on
  // B200 at M = 512: N = 4096, K = 11008 took 47.0 us against 61.6 us on
  // 128 x 128 tiles, while K = 4096 (28.6 against 26.6 us) and the two-wave
  // shapes N = 12288 and 22016 at K = 4096 (65.7 / 97.5 against 58.6 / 86.5 us
  // unsplit) were slower.
  const int num_k = (K + BK - 1) / BK;
  const bool can_split = split && split->ws && split->sync && tpair <= split->tiles &&
                         tpair <= gemm_split_max_tiles(num_sms) && num_k >= 8;
  const double esplit = can_split ? eff(2 * tpair, num_sms / 2, 0.35 + 12.0 / num_k) : 1e30;
  const int splits = esplit < epair ? 2 : 1;
  if (splits == 2) epair = esplit;
  if (b_tiled && N % 256 == 0 && num_sms >= 2 && epair < e128 && epair < e256) {
    CUtensorMap mb;
    if (bmap)
      mb = *bmap;  // the library's weights: encoded once when they were set
    else if (!make_tmap_weights(&mb, B, 1, N, K, 128))
      return cudaErrorInvalidValue;
    return launch_tc_pair(A, mb, M, N, K, ep, num_sms, st, splits, splits > 1 ? split->ws : nullptr,
                          splits > 1 ? split->sync : nullptr);
  }
  const bool use256 = (N % 256 == 0) && e256 <= e128 * 1.05;
  return use256 ? launch_tc<256>(A, B, b_tiled, M, N, K, ep, num_sms, st, bmap)
                : launch_tc<128>(A, B, b_tiled, M, N, K, ep, num_sms, st, bmap);
}

}  // namespace llama
