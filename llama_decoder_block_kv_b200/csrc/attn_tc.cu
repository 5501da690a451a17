// Causal grouped-query prefill attention on the 5th-generation tensor cores.
//
// What is computed: for the query of sequence b at position
// p = start_pos[b] + s and query head h,
// softmax_j(q.k_j / sqrt(D)) over the cached keys j <= p of kv head h / n_rep,
// times V ("LLaMA: Open and Efficient Foundation Language Models" notes,
// Attention.forward and repeat_kv; "灵哥讲llama3(中)", the cached-mask comment).
//
// One CTA owns 128 query rows of one (sequence, kv head): hpc query heads of
// that group x 128/hpc consecutive positions (row r = position r / hpc, head
// r % hpc), so every K/V tile is loaded once for those heads. hpc is the
// largest power of two (at most 8) dividing n_rep, so the rows hold whole
// positions and a kv head's n_rep query heads take n_rep / hpc CTAs.
//   warp 0      TMA: the Q tile once (a 3-D box over [token][head][d]), then
//               64-key K and V tiles of the cache into a 3-stage ring;
//   warp 1      TMEM owner and MMA issuer: S(j) = Q K(j)^T into one of two
//               64-column TMEM buffers, and O += P(j-1) V(j-1) into a D-column
//               TMEM accumulator (P from shared memory, V read N-major);
//   warps 2..5  softmax, one thread per query row (its TMEM lane): read the
//               row of S, mask, exponentiate against a running maximum that is
//               raised only when a new score exceeds it by more than 2^8 (then
//               O and the sum are rescaled in TMEM), write P as bf16 into shared
//               memory; at the end O / sum -> bf16 output.
// S(j+1) is computed while the softmax of tile j runs. Key tiles beyond the
// block's last position are never loaded; the causal predicate masks the rest.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int KT = 64;       // keys per tile
constexpr int RING = 3;      // K/V stages
constexpr float LOG2E_TC = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;  // raise the running max only past 2^8
}  // namespace

template <int D>
struct AttnTcCfg {
  static constexpr int HALVES = D / 64;
  static constexpr uint32_t Q_BYTES = 128 * D * 2;   // two (or one) 128 x 64 boxes
  static constexpr uint32_t KV_BYTES = KT * D * 2;   // one K or one V tile
  static constexpr uint32_t P_BYTES = 128 * KT * 2;  // 128 rows x 64 keys (two buffers)
  static constexpr size_t SMEM = 1024 + Q_BYTES + RING * 2 * KV_BYTES + 2 * P_BYTES + 256;
  static constexpr uint32_t TMEM_COLS = 256;  // S0, S1 (64 columns each), O (D columns)
};

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// shared-memory descriptor, 128-byte swizzle, explicit leading/stride byte offsets
__device__ __forceinline__ uint64_t make_sw128_desc_lbo(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// 2^x on the special-function unit (inputs below -126 give 0; -inf gives 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                           const __grid_constant__ CUtensorMap map_v, bf16* __restrict__ o,
                           const int* __restrict__ start_pos, int sp_scalar, int T, int H, int Hkv, int S_max,
                           int hpc, int* err) {
  using Cfg = AttnTcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sKV = sQ + Cfg::Q_BYTES;                 // RING x (K, V)
  uint8_t* sP = sKV + RING * 2 * Cfg::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * Cfg::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;          // [RING]
  uint64_t* kv_empty = kv_full + RING;   // [RING]
  uint64_t* s_full = kv_empty + RING;    // [2]
  uint64_t* s_free = s_full + 2;         // [2]
  uint64_t* p_full = s_free + 2;         // [2] per P buffer
  uint64_t* o_done = p_full + 2;         // [2] PV(j) completes o_done[j & 1]
  uint64_t* drained = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rep = H / Hkv, groups = n_rep / hpc;
  const int BQ = 128 / hpc;
  const int qblk = gridDim.x - 1 - blockIdx.x;  // longest (latest) query blocks first
  const int z = blockIdx.y;
  const int b = z / (Hkv * groups);
  const int kvh = (z / groups) % Hkv;
  const int grp = z % groups;
  const int h0 = kvh * n_rep + grp * hpc;
  const int q0 = qblk * BQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < RING; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const int sp = start_pos ? start_pos[b] : sp_scalar;
  const int q_last = min(q0 + BQ, T) - 1;
  const int kv_len = min(sp + q_last + 1, S_max);
  const int n = (kv_len + KT - 1) / KT;
  const int row0 = (b * Hkv + kvh) * S_max;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      prefetch_tensormap(&map_q);
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      mbar_arrive_expect_tx(q_full, Cfg::Q_BYTES);
#pragma unroll
      for (int hf = 0; hf < Cfg::HALVES; ++hf)
        tma_load_3d(sQ + hf * 16384, &map_q, q_full, hf * 64, h0, b * T + q0);
      int j = 0;
      for (; j < n; ++j) {
        const int st = j % RING;
        if (!wait_or_abort(&kv_empty[st], ((j / RING) & 1) ^ 1, err, abort_flag)) break;
        uint8_t* k_dst = sKV + st * 2 * Cfg::KV_BYTES;
        uint8_t* v_dst = k_dst + Cfg::KV_BYTES;
        mbar_arrive_expect_tx(&kv_full[st], 2 * Cfg::KV_BYTES);
#pragma unroll
        for (int hf = 0; hf < Cfg::HALVES; ++hf) {
          tma_load_2d(k_dst + hf * 8192, &map_k, &kv_full[st], hf * 64, row0 + j * KT);
          tma_load_2d(v_dst + hf * 8192, &map_v, &kv_full[st], hf * 64, row0 + j * KT);
        }
      }
      // every copy into this CTA's shared memory lands before the CTA can retire
      mbar_wait(q_full, 0, err);
      for (int i = (j > RING ? j - RING : 0); i < j; ++i) mbar_wait(&kv_full[i % RING], (i / RING) & 1, err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = make_idesc_bf16(128, KT);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D) | (1u << 16);  // B (= V) N-major
      const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
      bool ok = wait_or_abort(q_full, 0, err, abort_flag);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % RING;
          if (!wait_or_abort(&kv_full[st], (j / RING) & 1, err, abort_flag)) break;
          if (!wait_or_abort(&s_free[j & 1], ((j >> 1) & 1) ^ 1, err, abort_flag)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + st * 2 * Cfg::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;   // Q: 16 KB per 64-wide half
            const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;   // K: 8 KB per half
            tc_mma_bf16(tmem + (j & 1) * KT, make_sw128_desc(q_addr + off), make_sw128_desc(k_addr + koff), idesc_s,
                        kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[j & 1]);
        }
        if (j >= 1) {
          const int jp = j - 1, stp = jp % RING;
          if (!wait_or_abort(&p_full[jp & 1], (jp >> 1) & 1, err, abort_flag)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sKV + stp * 2 * Cfg::KV_BYTES + Cfg::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk) {
            // A = P (K-major: 128 rows x 64 keys); B = V N-major: 16 keys (2048 B) per step,
            // 64-wide d blocks 8 KB apart (leading byte offset), 8-key groups 1 KB apart
            tc_mma_bf16(tmem + 2 * KT, make_sw128_desc(p_addr + (jp & 1) * Cfg::P_BYTES + kk * 32),
                        make_sw128_desc_lbo(v_addr + kk * 2048, 8192, 1024), idesc_pv, (jp | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&o_done[jp & 1]);
          tc_commit(&kv_empty[stp]);
        }
      }
      tc_commit(drained);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drained, 0) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
      }
    }
  } else {
    // -------------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // query row = TMEM lane
    const int pos_l = r / hpc, hl = r - pos_l * hpc;
    const int p_row = sp + min(q0 + pos_l, T - 1);
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = rsqrtf((float)D) * LOG2E_TC;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = wait_or_abort(&s_full[j & 1], (j >> 1) & 1, err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[KT];
      tmem_ld_32cols(lane_base + (j & 1) * KT, s);
      tmem_ld_32cols(lane_base + (j & 1) * KT + 32, s + 32);
      tc_fence_before();
      mbar_arrive(&s_free[j & 1]);
      // row maximum of the raw scores (masked keys -inf), four independent chains
      const int key0 = j * KT;
      if (__any_sync(0xffffffffu, key0 + KT - 1 > p_row)) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (key0 + c > p_row) s[c] = -INFINITY;
      }
      float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < KT; c += 4) {
        mx[0] = fmaxf(mx[0], s[c]);
        mx[1] = fmaxf(mx[1], s[c + 1]);
        mx[2] = fmaxf(mx[2], s[c + 2]);
        mx[3] = fmaxf(mx[3], s[c + 3]);
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;  // log2 units
      // P(j) goes to buffer j & 1, last read by PV(j-2)
      if (j >= 2) {
        ok = wait_or_abort(&o_done[j & 1], ((j - 2) >> 1) & 1, err, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (j == 0) {
        m_used = mt;
      } else if (__any_sync(0xffffffffu, mt > m_used + RESCALE_LOG2)) {
        // O is rescaled in TMEM only once PV(j-1) has finished accumulating into it
        ok = wait_or_abort(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, err, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float m_new = fmaxf(m_used, mt);
        const float alpha = exp2f(m_used - m_new);
        l *= alpha;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float ov[32];
          tmem_ld_32cols(lane_base + 2 * KT + c, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tmem_st_32cols(lane_base + 2 * KT + c, ov);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        m_used = m_new;
      }
      // P row -> bf16 in the 128-byte-swizzled K-major layout the MMA reads;
      // p = 2^(s * log2(e)/sqrt(D) - m) is one FMA and one ex2
      uint8_t* prow = sP + (j & 1) * Cfg::P_BYTES + r * 128;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c8 = 0; c8 < KT / 8; ++c8) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = ex2_approx(fmaf(s[c8 * 8 + e], sl2, -m_used));
          ls[e & 3] += pv[e];
        }
        uint4 u;
        u.x = pack_bf16x2(pv[0], pv[1]);
        u.y = pack_bf16x2(pv[2], pv[3]);
        u.z = pack_bf16x2(pv[4], pv[5]);
        u.w = pack_bf16x2(pv[6], pv[7]);
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) = u;
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    if (ok) {
      ok = wait_or_abort(&o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
      const bool store = q0 + pos_l < T;
      bf16* dst = o + ((size_t)(b * T + q0 + pos_l) * H + h0 + hl) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld_32cols(lane_base + 2 * KT + c, ov);
        if (store) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float v8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v8[i] = ov[e + i] * inv;
            store8(dst + c + e, v8);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// 3-D bf16 tensor map over q [tokens][H][D] with a box of 64 d x hpc heads x
// (128 / hpc) tokens and 128-byte swizzling: the box lands as 128 rows of 128 B
// ordered (token, head), the canonical K-major tile of the MMA.
static bool make_q_map(CUtensorMap* map, const void* q, int tokens, int H, int D, int hpc);

template <int D>
static cudaError_t prefill_tc_d(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, const int* sp,
                                int sp_scalar, int B, int T, int H, int Hkv, int S_max, int* err, cudaStream_t st) {
  const int n_rep = H / Hkv;
  const int hpc = prefill_heads_per_cta(n_rep);
  const int BQ = 128 / hpc;
  CUtensorMap mq;
  if (!make_q_map(&mq, q, B * T, H, D, hpc)) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(attn_prefill_tc_kernel<D>, AttnTcCfg<D>::SMEM, attr);
  if (e != cudaSuccess) return e;
  dim3 grid((T + BQ - 1) / BQ, B * Hkv * (n_rep / hpc));
  return launch_pdl(attn_prefill_tc_kernel<D>, grid, dim3(192), AttnTcCfg<D>::SMEM, st, mq, mk, mv,
                    reinterpret_cast<bf16*>(o), sp, sp_scalar, T, H, Hkv, S_max, hpc, err);
}

cudaError_t launch_attn_prefill_tc(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o,
                                   const int* sp, int sp_scalar, int B, int T, int H, int Hkv, int D, int S_max,
                                   int* err, cudaStream_t st) {
  if (D == 128) return prefill_tc_d<128>(mk, mv, q, o, sp, sp_scalar, B, T, H, Hkv, S_max, err, st);
  return prefill_tc_d<64>(mk, mv, q, o, sp, sp_scalar, B, T, H, Hkv, S_max, err, st);
}

static bool make_q_map(CUtensorMap* map, const void* q, int tokens, int H, int D, int hpc) {
  return make_tmap_bf16_3d(map, q, (uint64_t)D, (uint64_t)H, (uint64_t)tokens, 64, (uint32_t)hpc,
                           (uint32_t)(128 / hpc));
}

}  // namespace llama
