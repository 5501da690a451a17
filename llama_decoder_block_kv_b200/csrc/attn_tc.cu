// Causal grouped-query prefill attention on the 5th-generation tensor cores,
// issued by CTA pairs with the 2-SM MMA form.
//
// What is computed: for the query of sequence b at position
// p = start_pos[b] + s and query head h,
// softmax_j(q.k_j / sqrt(D)) over the cached keys j <= p of kv head h / n_rep,
// times V ("LLaMA: Open and Efficient Foundation Language Models" notes,
// Attention.forward and repeat_kv; "灵哥讲llama3(中)", the cached-mask comment).
//
// A CTA owns 128 query rows of one (sequence, kv head): hpc query heads of
// that group x 128/hpc consecutive positions (row r = position r / hpc, head
// r % hpc). hpc is the largest power of two (at most 8) dividing n_rep, so
// the rows hold whole positions. Two CTAs of a cluster (ranks 0 and 1, on an
// SM pair) take two consecutive query blocks of the same (sequence, kv head,
// head group), 256 rows, and share every MMA: the rank-0 CTA issues
// tcgen05.mma.cta_group::2 with M = 256, each CTA supplying its 128 rows of A
// and half of B from its own shared memory (or TMEM), and each CTA's TMEM
// receiving its 128 rows of the result. On B200 one such instruction costs
// about as long as the 1-SM form for 128 rows (~70 cycles at N = 128 against
// ~125 for the 1-SM form, measured), so the MMA time per row halves.
//   warp 0      TMA, in each CTA, into its own shared memory: its Q tile once
//               (a 3-D box over [token][head][d]), then its halves of the
//               128-key K tiles (keys 64 r .. 64 r + 63 of the tile, both d
//               halves) and of the V tiles (d half r, all 128 keys), three
//               stages each. The copies of both CTAs complete on rank 0's
//               barriers (the 2-SM copy form), which rank 0 primes with both
//               halves' bytes;
//   warp 1      both CTAs: TMEM (allocated for the pair). Rank 0, lane 0: the
//               P V issuer, O += P(j) V(j) with P read from each CTA's TMEM,
//               where its softmax wrote it over S(j). Rank 1, lane 0: relays
//               "P(j) written" in its CTA to rank 0's P barrier (a remote
//               arrival);
//   warp 6      rank 0, lane 0: the S issuer, S(j) = Q K(j)^T into TMEM buffer
//               j mod 3 (128 columns) as soon as K(j) is in and the buffer's
//               previous P V has finished. Two issuing threads keep the tensor
//               pipe fed: it takes one 2-SM MMA per ~70 cycles and queues few,
//               so a wait in one issuer would otherwise idle it. Every commit
//               arrives on the barriers of both CTAs;
//   warps 2..5  softmax, one thread per query row of the CTA (its TMEM lane; a
//               warp reaches only the lanes of its quarter, warp id mod 4). A
//               thread reads its row of S, masks it, raises its running maximum
//               only when a score exceeds it by more than 2^8 (O and the sum
//               are then rescaled in TMEM), and writes P over S as two bf16
//               parts (P = P_hi + P_lo, the second the rounding of the
//               remainder), so O += P_hi V + P_lo V keeps about 16 bits of each
//               probability. At the end O / (sum of P) -> bf16.
// A buffer holds S(j), then P(j), until P(j) V(j) has finished; S(j + 3) waits
// for that (pv_done). Key tiles beyond the pair's last position are never
// loaded; the causal predicate masks the rest (the earlier block of a pair
// masks the keys past its own rows).
//
// attn_prefill_tc_kernel, further down, is the single-CTA form: one CTA per
// 128 rows, the 1-SM MMA form, one issuing thread. It runs head_dim 64 (its V
// tile's 64 d columns are one TMA box, which the pair's N split would halve)
// and short calls, where the pair's longer start and end cost more than its
// faster MMAs save.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int KT = 128;      // keys per tile
constexpr int NBUF = 3;      // S / P buffers in TMEM
constexpr int KRING = 2;     // K stages (a K tile is free once S(j) is computed)
constexpr int VRING = 3;     // V stages (a V tile is free once P(j) V(j) is computed)
constexpr float LOG2E_TC = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;  // raise the running max only past 2^8
}  // namespace

template <int D>
struct AttnTcCfg {
  static constexpr int HALVES = D / 64;
  static constexpr uint32_t Q_BYTES = 128 * D * 2;      // two (or one) 128 x 64 boxes
  static constexpr uint32_t HALF_BYTES = KT * 128;      // 128 keys x 64 d of bf16 (two 64-row boxes)
  static constexpr uint32_t KV_BYTES = HALVES * HALF_BYTES;  // one K or one V tile
  static constexpr size_t SMEM = 1024 + Q_BYTES + (KRING + VRING) * KV_BYTES + 512;
  // three 128-column S buffers (P(j) is written over S(j): 64 columns of bf16
  // pairs for P_hi, then 64 for P_lo), then O (D columns)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t P_LO_COL = KT / 2;
  static constexpr uint32_t O_COL = NBUF * KT;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
};

// The CTA-pair kernel: each CTA holds its own Q, half of each K tile (64 keys,
// every d) and half of each V tile (one 64-wide d half, all 128 keys)
template <int D>
struct PairCfg {
  static_assert(D == 128, "the pair kernel splits V's head dimension into two 64-wide halves");
  static constexpr int HALVES = D / 64;
  static constexpr uint32_t Q_BYTES = 128 * D * 2;
  static constexpr uint32_t KBOX = 64 * 128;             // 64 keys x 64 d of bf16 (one TMA box)
  static constexpr uint32_t K_BYTES = HALVES * KBOX;     // this CTA's 64 keys of a K tile
  static constexpr uint32_t V_BYTES = 2 * KBOX;          // this CTA's d half of a V tile
  static constexpr int K_STAGES = 3;                     // K, V and S/P buffers all three deep
  static constexpr size_t SMEM = 1024 + Q_BYTES + K_STAGES * K_BYTES + VRING * V_BYTES + 512;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t P_LO_COL = KT / 2;
  static constexpr uint32_t O_COL = NBUF * KT;
};

// D[tmem] (+)= A[tmem] * B[smem]: A = 128 rows (TMEM lanes) x 16 bf16 (8 columns of
// bf16 pairs, K-major), B by shared-memory descriptor, fp32 accumulation.
__device__ __forceinline__ void tc_mma_bf16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// NC consecutive TMEM columns of this thread's lane: NC / 32 loads, one wait
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
  uint32_t r[NC];
#pragma unroll
  for (int h = 0; h < NC / 32; ++h)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[32 * h + 0]), "=r"(r[32 * h + 1]), "=r"(r[32 * h + 2]), "=r"(r[32 * h + 3]),
          "=r"(r[32 * h + 4]), "=r"(r[32 * h + 5]), "=r"(r[32 * h + 6]), "=r"(r[32 * h + 7]),
          "=r"(r[32 * h + 8]), "=r"(r[32 * h + 9]), "=r"(r[32 * h + 10]), "=r"(r[32 * h + 11]),
          "=r"(r[32 * h + 12]), "=r"(r[32 * h + 13]), "=r"(r[32 * h + 14]), "=r"(r[32 * h + 15]),
          "=r"(r[32 * h + 16]), "=r"(r[32 * h + 17]), "=r"(r[32 * h + 18]), "=r"(r[32 * h + 19]),
          "=r"(r[32 * h + 20]), "=r"(r[32 * h + 21]), "=r"(r[32 * h + 22]), "=r"(r[32 * h + 23]),
          "=r"(r[32 * h + 24]), "=r"(r[32 * h + 25]), "=r"(r[32 * h + 26]), "=r"(r[32 * h + 27]),
          "=r"(r[32 * h + 28]), "=r"(r[32 * h + 29]), "=r"(r[32 * h + 30]), "=r"(r[32 * h + 31])
        : "r"(taddr + 32 * h)
        : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < NC; ++i) v[i] = __uint_as_float(r[i]);
}

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

// sm_100 packed fp32 arithmetic: two lanes of a 64-bit register per instruction
// (halves the FMA-pipe instructions of the softmax), and the 3-input maximum.
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub_f2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

constexpr int SOFTMAX_THREADS = 128;  // 4 warps, one thread per query row (its TMEM lane)
constexpr int ATTN_TC_THREADS = 64 + SOFTMAX_THREADS;

template <int D>
__global__ void __launch_bounds__(ATTN_TC_THREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                           const __grid_constant__ CUtensorMap map_v, bf16* __restrict__ o,
                           const int* __restrict__ start_pos, int sp_scalar, int T, int H, int Hkv, int S_max,
                           int hpc, int* err) {
  using Cfg = AttnTcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + Cfg::Q_BYTES;                  // KRING K tiles
  uint8_t* sV = sK + KRING * Cfg::KV_BYTES;         // VRING V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VRING * Cfg::KV_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;           // [KRING]
  uint64_t* k_empty = k_full + KRING;    // [KRING]
  uint64_t* v_full = k_empty + KRING;    // [VRING]
  uint64_t* v_empty = v_full + VRING;    // [VRING]
  uint64_t* s_full = v_empty + VRING;    // [NBUF] buffer j % NBUF holds S(j)
  uint64_t* p_full = s_full + NBUF;      // [NBUF] ... then P(j), written over it
  uint64_t* s_free = p_full + NBUF;      // [NBUF] ... and P(j) V(j), which read it, has finished
  uint64_t* drained = s_free + NBUF;     // every MMA of the CTA has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rep = H / Hkv, groups = n_rep / hpc;
  const int BQ = 128 / hpc;
  // blocks are dispatched in linear order (x fastest): the query-block index is
  // the slow dimension, counted down, so the longest (latest) query blocks of
  // every head start first and the short ones fill the tail
  const int qblk = gridDim.y - 1 - blockIdx.y;
  const int z = blockIdx.x;
  const int b = z / (Hkv * groups);
  const int kvh = (z / groups) % Hkv;
  const int grp = z % groups;
  const int h0 = kvh * n_rep + grp * hpc;
  const int q0 = qblk * BQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < KRING; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < VRING; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], SOFTMAX_THREADS);
      mbar_init(&s_free[i], 1);
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
      // a 128-key tile of one d half is two 64-row boxes, back to back: 128 rows
      // of 128 B in the swizzled layout both MMAs read (rows past the tensor's
      // end arrive as zeros; rows past the block's keys are masked)
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int t) {
        mbar_arrive_expect_tx(bar, Cfg::KV_BYTES);
#pragma unroll
        for (int hf = 0; hf < Cfg::HALVES; ++hf)
#pragma unroll
          for (int kh = 0; kh < 2; ++kh)
            tma_load_2d(dst + hf * Cfg::HALF_BYTES + kh * 8192, map, bar, hf * 64, row0 + t * KT + kh * 64);
      };
      // K(t) waits for S(t - KRING); V(j) for P(j - VRING) V(j - VRING)
      auto load_k = [&](int t) -> bool {
        const int st = t % KRING;
        if (!wait_or_abort(&k_empty[st], ((t / KRING) & 1) ^ 1, err, abort_flag)) return false;
        load_tile(&map_k, sK + st * Cfg::KV_BYTES, &k_full[st], t);
        return true;
      };
      int nk_issued = 0, nv_issued = 0;
      bool ok = true;
      for (; ok && nk_issued < min(n, KRING); ++nk_issued) ok = load_k(nk_issued);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % VRING;
        if (!(ok = wait_or_abort(&v_empty[st], ((j / VRING) & 1) ^ 1, err, abort_flag))) break;
        load_tile(&map_v, sV + st * Cfg::KV_BYTES, &v_full[st], j);
        ++nv_issued;
        if (nk_issued < n && (ok = load_k(nk_issued))) ++nk_issued;
      }
      // every copy into this CTA's shared memory lands before the CTA can retire
      mbar_wait(q_full, 0, err);
      for (int i = (nk_issued > KRING ? nk_issued - KRING : 0); i < nk_issued; ++i)
        mbar_wait(&k_full[i % KRING], (i / KRING) & 1, err);
      for (int i = (nv_issued > VRING ? nv_issued - VRING : 0); i < nv_issued; ++i)
        mbar_wait(&v_full[i % VRING], (i / VRING) & 1, err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = make_idesc_bf16(128, KT);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D) | (1u << 16);  // B (= V) N-major
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = wait_or_abort(q_full, 0, err, abort_flag);
      // S(j) = Q K(j)^T into buffer j % NBUF once K(j) is in and P(j - NBUF) V(j - NBUF),
      // which read that buffer last, has finished
      auto issue_s = [&](int js) -> bool {
        const int st = js % KRING, sb = js % NBUF;
        if (!wait_or_abort(&k_full[st], (js / KRING) & 1, err, abort_flag)) return false;
        if (!wait_or_abort(&s_free[sb], ((js / NBUF) & 1) ^ 1, err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * Cfg::KV_BYTES);
        const uint32_t sd = tmem + (uint32_t)(sb * KT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;              // Q: 16 KB per 64-wide half
          const uint32_t koff = (kk >> 2) * Cfg::HALF_BYTES + (kk & 3) * 32;   // K: 128 rows per half
          tc_mma_bf16(sd, make_sw128_desc(q_addr + off), make_sw128_desc(k_addr + koff), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        tc_commit(&k_empty[st]);
        return true;
      };
      // Order: S(0), then S(j + 1), PV(j) for each j: S(j + 1) waits for PV(j - 2),
      // issued two steps earlier, and the softmax of tile j + 1 runs under PV(j).
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;
        const int sb = j % NBUF, st = j % VRING;
        if (!(ok = wait_or_abort(&v_full[st], (j / VRING) & 1, err, abort_flag))) break;
        if (!(ok = wait_or_abort(&p_full[sb], (j / NBUF) & 1, err, abort_flag))) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * Cfg::KV_BYTES);
        const uint32_t od = tmem + Cfg::O_COL;
        const uint32_t pa = tmem + (uint32_t)(sb * KT);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          // A = P from TMEM (128 lanes x 16 keys = 8 columns of bf16 pairs per step);
          // B = V N-major: 16 keys (2048 B) per step, 64-wide d halves HALF_BYTES
          // apart (leading byte offset), 8-key groups 1 KB apart.
          // O += P_hi V + P_lo V: P carries ~16 significant bits into the sum.
          const uint64_t vdesc = make_sw128_desc_lbo(v_addr + kk * 2048, Cfg::HALF_BYTES, 1024);
          tc_mma_bf16_tmem_a(od, pa + kk * 8, vdesc, idesc_pv, (j | kk) != 0 ? 1u : 0u);
          tc_mma_bf16_tmem_a(od, pa + Cfg::P_LO_COL + kk * 8, vdesc, idesc_pv, 1u);
        }
        tc_commit(&s_free[sb]);
        tc_commit(&v_empty[st]);
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
    const uint32_t o_cols = lane_base + Cfg::O_COL;
    const float sl2 = rsqrtf((float)D) * LOG2E_TC;
    const uint64_t scale2 = f2(sl2, sl2);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j % NBUF;
      ok = wait_or_abort(&s_full[sb], (j / NBUF) & 1, err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_cols = lane_base + sb * KT;
      float s[KT];
      tmem_ld_cols<KT>(s_cols, s);
      // row maximum of the raw scores (masked keys -inf): four chains of 3-input maxima
      const int key0 = j * KT;
      if (__any_sync(0xffffffffu, key0 + KT - 1 > p_row)) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (key0 + c > p_row) s[c] = -INFINITY;
      }
      float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < KT; c += 8)
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;  // log2 units
      if (j == 0) {
        m_used = mt;
      } else if (__any_sync(0xffffffffu, mt > m_used + RESCALE_LOG2)) {
        // rescale O in TMEM once P(j - 1) V(j - 1) has finished (S(j) being here means
        // P(j - 1 - NBUF) V(j - 1 - NBUF), the previous use of that buffer, has, so the
        // phase waited for is the latest one or the next)
        const int pb = (j - 1) % NBUF;
        ok = wait_or_abort(&s_free[pb], ((j - 1) / NBUF) & 1, err, abort_flag);
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
          tmem_ld_32cols(o_cols + c, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tmem_st_32cols(o_cols + c, ov);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        m_used = m_new;
      }
      // P row -> bf16 pairs written over this row's S in TMEM (column c holds keys
      // 2c, 2c + 1, the K-major A layout of the PV MMA); P_lo P_LO_COL columns on.
      // p = 2^(s * log2(e)/sqrt(D) - m): one packed FMA per pair and one ex2 each.
      // (Key 0 is visible to every row, so m_used is finite from the first tile;
      // the guard keeps 2^(-inf - m) = 0 meaningful all the same.)
      const float m_ref = m_used == -INFINITY ? 0.f : m_used;
      const uint64_t negm2 = f2(-m_ref, -m_ref);
      uint64_t lsum[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < KT / 64; ++h) {
        float ph[32], plo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float t0, t1;
          f2_split(fma_f2(f2(s[64 * h + 2 * e], s[64 * h + 2 * e + 1]), scale2, negm2), t0, t1);
          const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
          const uint64_t p2 = f2(p0, p1);
          lsum[e & 1] = add_f2(lsum[e & 1], p2);
          const uint32_t hi = pack_bf16x2(p0, p1);
          ph[e] = __uint_as_float(hi);
          // lo = bf16(p - hi), the remainder taken as one packed subtraction
          float r0, r1;
          f2_split(sub_f2(p2, f2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xFFFF0000u))), r0, r1);
          plo[e] = __uint_as_float(pack_bf16x2(r0, r1));
        }
        tmem_st_32cols(s_cols + 32 * h, ph);
        tmem_st_32cols(s_cols + Cfg::P_LO_COL + 32 * h, plo);
      }
      {
        float a0, a1, b0, b1;
        f2_split(lsum[0], a0, a1);
        f2_split(lsum[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    // every MMA of the CTA has finished (the MMA thread commits `drained` once,
    // after its last PV), so O is complete
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(drained, 0, err, abort_flag));
    if (ok) {
      // O / l -> bf16
      tc_fence_after();
      const float inv = 1.f / l;
      const bool store = q0 + pos_l < T;
      bf16* dst = o + ((size_t)(b * T + q0 + pos_l) * H + h0 + hl) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld_32cols(o_cols + c, ov);
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

// ---------------------------------------------------------------- CTA-pair kernel
constexpr int PAIR_THREADS = 64 + SOFTMAX_THREADS + 32;  // + warp 6: rank 0's S issuer

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    attn_prefill_pair_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                             const __grid_constant__ CUtensorMap map_v, bf16* __restrict__ o,
                             const int* __restrict__ start_pos, int sp_scalar, int T, int H, int Hkv, int S_max,
                             int hpc, int* err) {
  using Cfg = PairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + Cfg::Q_BYTES;                  // NBUF halves of K tiles
  uint8_t* sV = sK + NBUF * Cfg::K_BYTES;          // NBUF halves of V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NBUF * Cfg::V_BYTES);
  uint64_t* q_full = bars;                      // both CTAs' Q landed (rank 0's barrier, both copies)
  // K(t) / V(t) landed in both CTAs: rank 0's barrier, which the copies of both
  // CTAs complete (the 2-SM copy form) and rank 0 expects both halves' bytes on.
  // Stage, S buffer and ring indices are all t % 3.
  uint64_t* k_full = q_full + 1;                // [3]
  uint64_t* v_full = k_full + NBUF;             // [3]
  uint64_t* s_done = v_full + NBUF;             // [3] S(j) finished: S ready, K stage free (commit to both)
  uint64_t* pv_done = s_done + NBUF;            // [3] P(j) V(j) finished: buffer and V stage free (commit to both)
  // [3] P(j) written over S(j): this CTA's 128 softmax threads, and on rank 0
  // one more arrival relayed from rank 1 once its P(j) is written
  uint64_t* p_full = pv_done + NBUF;
  uint64_t* drained = p_full + NBUF;            // every MMA of both issuers has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_rep = H / Hkv, groups = n_rep / hpc;
  const int BQ = 128 / hpc;
  // the pair index is the slow dimension, counted down: the longest pairs start first
  const int pair = gridDim.y - 1 - blockIdx.y;
  const int z = blockIdx.x >> 1;
  const int b = z / (Hkv * groups);
  const int kvh = (z / groups) % Hkv;
  const int grp = z % groups;
  const int h0 = kvh * n_rep + grp * hpc;
  const int q0 = (2 * pair + (int)rank) * BQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&s_done[i], 1);
      mbar_init(&pv_done[i], 1);
      mbar_init(&p_full[i], SOFTMAX_THREADS + (rank == 0 ? 1 : 0));
    }
    mbar_init(drained, 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // TMEM for the pair: the same warp of both CTAs allocates
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival or commit
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const int sp = start_pos ? start_pos[b] : sp_scalar;
  const int q_last = min((2 * pair + 2) * BQ, T) - 1;  // the pair's last position
  const int kv_len = min(sp + q_last + 1, S_max);
  const int n = (kv_len + KT - 1) / KT;
  const int row0 = (b * Hkv + kvh) * S_max;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer (both CTAs)
      prefetch_tensormap(&map_q);
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      // this CTA's Q tile, completing on rank 0's q_full (primed with both tiles' bytes)
      if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * Cfg::Q_BYTES);
      {
        const uint32_t bar = mbar_cluster_addr(q_full, 0);
#pragma unroll
        for (int hf = 0; hf < Cfg::HALVES; ++hf)
          tma_load_3d_pair(sQ + hf * 16384, &map_q, bar, hf * 64, h0, b * T + q0);
      }
      // K(t): keys 64 rank .. 64 rank + 63 of the tile, every d half, into this
      // CTA; the bytes complete on rank 0's k_full, which rank 0 primes with both
      // halves. Waits for S(t - 3).
      auto load_k = [&](int t) -> bool {
        const int st = t % NBUF;
        if (!wait_or_abort(&s_done[st], ((t / NBUF) & 1) ^ 1, err, abort_flag)) return false;
        if (rank == 0) mbar_arrive_expect_tx(&k_full[st], 2 * Cfg::K_BYTES);
        const uint32_t bar = mbar_cluster_addr(&k_full[st], 0);
#pragma unroll
        for (int hf = 0; hf < Cfg::HALVES; ++hf)
          tma_load_2d_pair(sK + st * Cfg::K_BYTES + hf * Cfg::KBOX, &map_k, bar, hf * 64,
                           row0 + t * KT + (int)rank * 64);
        return true;
      };
      int nk_issued = 0, nv_issued = 0;
      bool ok = true;
      for (; ok && nk_issued < min(n, NBUF); ++nk_issued) ok = load_k(nk_issued);
      for (int j = 0; ok && j < n; ++j) {
        // V(j): d half `rank`, all 128 keys (two 64-key boxes), completing on rank
        // 0's v_full; waits for P(j - NBUF) V(j - NBUF)
        const int st = j % NBUF;
        if (!(ok = wait_or_abort(&pv_done[st], ((j / NBUF) & 1) ^ 1, err, abort_flag))) break;
        if (rank == 0) mbar_arrive_expect_tx(&v_full[st], 2 * Cfg::V_BYTES);
        const uint32_t bar = mbar_cluster_addr(&v_full[st], 0);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh)
          tma_load_2d_pair(sV + st * Cfg::V_BYTES + kh * Cfg::KBOX, &map_v, bar, (int)rank * 64,
                           row0 + j * KT + kh * 64);
        ++nv_issued;
        if (nk_issued < n && (ok = load_k(nk_issued))) ++nk_issued;
      }
      // every copy into either CTA's shared memory lands before the pair can
      // retire: rank 0's barriers count both CTAs' bytes, and rank 1 does not
      // pass the final cluster barrier before rank 0 has waited for them
      if (rank == 0) {
        mbar_wait(q_full, 0, err);
        for (int i = (nk_issued > NBUF ? nk_issued - NBUF : 0); i < nk_issued; ++i)
          mbar_wait(&k_full[i % NBUF], (i / NBUF) & 1, err);
        for (int i = (nv_issued > NBUF ? nv_issued - NBUF : 0); i < nv_issued; ++i)
          mbar_wait(&v_full[i % NBUF], (i / NBUF) & 1, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------------ PV issuer (rank 0)
      constexpr uint32_t idesc_pv = idesc2_bf16(256, D, true);  // B (= V) N-major
      // O += P(j) V(j) once V(j) is in both CTAs and both CTAs have written P(j)
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        const int sb = j % NBUF;
        if (!(ok = wait_or_abort(&v_full[sb], (j / NBUF) & 1, err, abort_flag))) break;
        if (!(ok = wait_cluster_or_abort(&p_full[sb], (j / NBUF) & 1, err, abort_flag))) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + sb * Cfg::V_BYTES);
        const uint32_t od = tmem + Cfg::O_COL;
        const uint32_t pa = tmem + (uint32_t)(sb * KT);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          // A = P from each CTA's TMEM (16 keys = 8 columns of bf16 pairs per step);
          // B = each CTA's d half of V, N-major: 16 keys (2048 B) per step, 8-key
          // groups 1 KB apart. O += P_hi V + P_lo V.
          const uint64_t vdesc = make_sw128_desc_lbo(v_addr + kk * 2048, Cfg::KBOX, 1024);
          mma2_ts(od, pa + kk * 8, vdesc, idesc_pv, (j | kk) != 0 ? 1u : 0u);
          mma2_ts(od, pa + Cfg::P_LO_COL + kk * 8, vdesc, idesc_pv, 1u);
        }
        commit2(&pv_done[sb]);
      }
      commit2(drained);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drained, 0) && global_timer_ns() - t0 < LLAMA_WAIT_LIMIT_NS) {
      }
    } else if (lane == 0) {
      // ------------------------------------------------------------------ forwarder (rank 1)
      // this CTA's "P(j) written", relayed onto rank 0's own P barrier as its one
      // arrival beyond the local threads'
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        if (!(ok = wait_or_abort(&p_full[j % NBUF], (j / NBUF) & 1, err, abort_flag))) break;
        mbar_arrive_remote_relaxed(&p_full[j % NBUF], 0);
      }
    }
  } else if (warp == 2 + SOFTMAX_THREADS / 32) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------------ S issuer (rank 0)
      // A second issuing thread: the tensor pipe takes one 2-SM MMA per ~70 cycles
      // and queues few, so while one issuer waits on a barrier the other keeps it fed.
      constexpr uint32_t idesc_s = idesc2_bf16(256, KT, false);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = wait_or_abort(q_full, 0, err, abort_flag);
      // S(j) = Q K(j)^T (M = 256: each CTA's Q; N = 128 keys: each CTA's half of K(j))
      // into buffer j % 3 once K(j) is in and P(j - 3) V(j - 3) has finished
      for (int js = 0; ok && js < n; ++js) {
        const int sb = js % NBUF;
        if (!(ok = wait_or_abort(&k_full[sb], (js / NBUF) & 1, err, abort_flag))) break;
        if (!(ok = wait_or_abort(&pv_done[sb], ((js / NBUF) & 1) ^ 1, err, abort_flag))) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + sb * Cfg::K_BYTES);
        const uint32_t sd = tmem + (uint32_t)(sb * KT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;         // Q: 16 KB per 64-wide half
          const uint32_t koff = (kk >> 2) * Cfg::KBOX + (kk & 3) * 32;    // K: 64 rows per d half
          mma2_ss(sd, make_sw128_desc(q_addr + off), make_sw128_desc(k_addr + koff), idesc_s, kk > 0 ? 1u : 0u);
        }
        commit2(&s_done[sb]);
      }
      commit2(drained);
    }
  } else {
    // -------------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // query row = TMEM lane
    const int pos_l = r / hpc, hl = r - pos_l * hpc;
    const int p_row = sp + min(q0 + pos_l, T - 1);
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t o_cols = lane_base + Cfg::O_COL;
    const float sl2 = rsqrtf((float)D) * LOG2E_TC;
    const uint64_t scale2 = f2(sl2, sl2);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j % NBUF;
      ok = wait_or_abort(&s_done[sb], (j / NBUF) & 1, err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_cols = lane_base + sb * KT;
      float s[KT];
      tmem_ld_cols<KT>(s_cols, s);
      // row maximum of the raw scores (masked keys -inf): four chains of 3-input maxima
      const int key0 = j * KT;
      if (__any_sync(0xffffffffu, key0 + KT - 1 > p_row)) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (key0 + c > p_row) s[c] = -INFINITY;
      }
      float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < KT; c += 8)
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;  // log2 units
      if (j == 0) {
        m_used = mt;
      } else if (__any_sync(0xffffffffu, mt > m_used + RESCALE_LOG2)) {
        // rescale O in TMEM once P(j - 1) V(j - 1) has finished (S(j) being here means
        // P(j - 1 - NBUF) V(j - 1 - NBUF), the previous use of that buffer, has, so the
        // phase waited for is the latest one or the next)
        const int pb = (j - 1) % NBUF;
        ok = wait_or_abort(&pv_done[pb], ((j - 1) / NBUF) & 1, err, abort_flag);
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
          tmem_ld_32cols(o_cols + c, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tmem_st_32cols(o_cols + c, ov);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        m_used = m_new;
      }
      // P row -> bf16 pairs written over this row's S in TMEM (column c holds keys
      // 2c, 2c + 1, the K-major A layout of the PV MMA); P_lo P_LO_COL columns on.
      // p = 2^(s * log2(e)/sqrt(D) - m): one packed FMA per pair and one ex2 each.
      // (Key 0 is visible to every row, so m_used is finite from the first tile;
      // the guard keeps 2^(-inf - m) = 0 meaningful all the same.)
      const float m_ref = m_used == -INFINITY ? 0.f : m_used;
      const uint64_t negm2 = f2(-m_ref, -m_ref);
      uint64_t lsum[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < KT / 64; ++h) {
        float ph[32], plo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float t0, t1;
          f2_split(fma_f2(f2(s[64 * h + 2 * e], s[64 * h + 2 * e + 1]), scale2, negm2), t0, t1);
          const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
          const uint64_t p2 = f2(p0, p1);
          lsum[e & 1] = add_f2(lsum[e & 1], p2);
          const uint32_t hi = pack_bf16x2(p0, p1);
          ph[e] = __uint_as_float(hi);
          // lo = bf16(p - hi), the remainder taken as one packed subtraction
          float r0, r1;
          f2_split(sub_f2(p2, f2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xFFFF0000u))), r0, r1);
          plo[e] = __uint_as_float(pack_bf16x2(r0, r1));
        }
        tmem_st_32cols(s_cols + 32 * h, ph);
        tmem_st_32cols(s_cols + Cfg::P_LO_COL + 32 * h, plo);
      }
      {
        float a0, a1, b0, b1;
        f2_split(lsum[0], a0, a1);
        f2_split(lsum[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    // every MMA of the CTA has finished (the MMA thread commits `drained` once,
    // after its last PV), so O is complete
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(drained, 0, err, abort_flag));
    if (ok) {
      // O / l -> bf16
      tc_fence_after();
      const float inv = 1.f / l;
      const bool store = q0 + pos_l < T;
      bf16* dst = o + ((size_t)(b * T + q0 + pos_l) * H + h0 + hl) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld_32cols(o_cols + c, ov);
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
  // the other CTA's shared memory and TMEM are read by the pair's MMAs until
  // `drained`, which both CTAs' softmax warps have waited for; neither CTA
  // frees its TMEM or retires before both get here
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::TMEM_COLS) : "memory");
  }
}

// 3-D bf16 tensor map over q [tokens][H][D] with a box of 64 d x hpc heads x
// (128 / hpc) tokens and 128-byte swizzling: the box lands as 128 rows of 128 B
// ordered (token, head), the canonical K-major tile of the MMA.
static bool make_q_map(CUtensorMap* map, const void* q, int tokens, int H, int D, int hpc);

template <int D>
static cudaError_t prefill_tc_d(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, const int* sp,
                                int sp_scalar, int B, int T, int H, int Hkv, int S_max, int* err, cudaStream_t st) {
  using Cfg = AttnTcCfg<D>;
  const int n_rep = H / Hkv;
  const int hpc = prefill_heads_per_cta(n_rep);
  const int BQ = 128 / hpc;
  CUtensorMap mq;
  if (!make_q_map(&mq, q, B * T, H, D, hpc)) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(attn_prefill_tc_kernel<D>, Cfg::SMEM, attr);
  if (e != cudaSuccess) return e;
  dim3 grid(B * Hkv * (n_rep / hpc), (T + BQ - 1) / BQ);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  return launch_pdl(attn_prefill_tc_kernel<D>, grid, dim3(ATTN_TC_THREADS), Cfg::SMEM, st, mq, mk, mv,
                    reinterpret_cast<bf16*>(o), sp, sp_scalar, T, H, Hkv, S_max, hpc, err);
}

// the shortest call (keys of its longest query) that runs the CTA-pair kernel
constexpr long long kPairMinKeys = 2048;

// CTA pairs (clusters of two) over pairs of consecutive query blocks
static cudaError_t prefill_pair(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, const int* sp,
                                int sp_scalar, int B, int T, int H, int Hkv, int S_max, int* err, cudaStream_t st) {
  using Cfg = PairCfg<128>;
  const int n_rep = H / Hkv;
  const int hpc = prefill_heads_per_cta(n_rep);
  const int BQ = 128 / hpc;
  CUtensorMap mq;
  if (!make_q_map(&mq, q, B * T, H, 128, hpc)) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(attn_prefill_pair_kernel<128>, Cfg::SMEM, attr);
  if (e != cudaSuccess) return e;
  const int blocks = (T + BQ - 1) / BQ;
  dim3 grid(2 * B * Hkv * (n_rep / hpc), (blocks + 1) / 2);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  return launch_pdl(attn_prefill_pair_kernel<128>, grid, dim3(PAIR_THREADS), Cfg::SMEM, st, mq, mk, mv,
                    reinterpret_cast<bf16*>(o), sp, sp_scalar, T, H, Hkv, S_max, hpc, err);
}

cudaError_t launch_attn_prefill_tc(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o,
                                   const int* sp, int sp_scalar, int B, int T, int H, int Hkv, int D, int S_max,
                                   int* err, cudaStream_t st) {
  // head_dim 128 and at least 2048 keys for the longest query (as far as the
  // host knows it: start_pos on the device counts as 0): CTA pairs sharing each
  // MMA, measured faster from there on (T = 4096 on the 7B layer 200 against
  // 221 us, T = 8192 on the 8B layer 0.655 against 0.783 ms; equal at 2048);
  // shorter calls, and head_dim 64 (V's 64-wide TMA box does not split in
  // two): one CTA per 128 rows
  const long long keys = (long long)(sp ? 0 : sp_scalar) + T;
  if (D == 128 && keys >= kPairMinKeys)
    return prefill_pair(mk, mv, q, o, sp, sp_scalar, B, T, H, Hkv, S_max, err, st);
  if (D == 128) return prefill_tc_d<128>(mk, mv, q, o, sp, sp_scalar, B, T, H, Hkv, S_max, err, st);
  return prefill_tc_d<64>(mk, mv, q, o, sp, sp_scalar, B, T, H, Hkv, S_max, err, st);
}

static bool make_q_map(CUtensorMap* map, const void* q, int tokens, int H, int D, int hpc) {
  return make_tmap_bf16_3d(map, q, (uint64_t)D, (uint64_t)H, (uint64_t)tokens, 64, (uint32_t)hpc,
                           (uint32_t)(128 / hpc));
}

}  // namespace llama
