// Causal grouped-query attention over the KV-cache.
//
// What is computed ("LLaMA: Open and Efficient Foundation Language Models"
// notes, Attention.forward and Transformer.forward; "灵哥讲llama3(中)", the
// cached-mask comment): for the query of sequence b at position
// p = start_pos[b] + s and query head h, attend over the cached keys
// j = 0 .. p of kv head h / n_rep (repeat_kv maps kv head j to query heads
// j*n_rep .. j*n_rep + n_rep - 1) with scores q.k / sqrt(D) and a softmax.
// The additive mask of the pages is never built: the predicate j <= p is
// applied inside the kernels and key tiles past the last position are never
// read (the pages' xformers remark: masked scores are not computed).
//
// Kernels (the prefill attention, T > 1, is the tcgen05 kernel of attn_tc.cu):
//  - attn_decode_kernel (T == 1): split-K flash decode. A CTA owns one
//    (sequence, kv head group, chunk of keys); the chunk streams through a
//    3-stage TMA ring (64-key K and V tiles, 128-byte swizzle, no multicast)
//    fed by a producer warp, the 4 compute warps each take 16 keys of every
//    64-key tile on the warp-level bf16 tensor-core MMA, their (max, sum, O)
//    states merge in shared memory and the CTA writes one partial; the CTA
//    that finishes last for a (sequence, head group) merges the partials of
//    all chunks with the log-sum-exp rule m = max m_c, l = sum l_c e^(m_c - m),
//    o = sum o_c e^(m_c - m) / l.
//  - attn_simple_kernel: fp32 mode (tiny models), one CTA per (token, head),
//    scores in shared memory, plain two-pass softmax.
#include "kernels.cuh"

#include <vector>

namespace llama {

namespace {
constexpr int KT = 64;  // keys per tile
constexpr float LOG2E = 1.4426950408889634f;
}  // namespace

// Byte address of element (row, col) inside a TMA box of 64 rows x 64 bf16
// written with 128-byte swizzling: the 16-byte chunk index is XOR-ed with row % 8.
__device__ __forceinline__ uint32_t sw_addr(uint32_t box_base, int row, int col) {
  return box_base + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

template <int D>
struct AttnSmem {
  static constexpr int HALVES = D / 64;
  static constexpr uint32_t TILE_BYTES = KT * D * 2;  // one K or one V tile
};

// Issue the TMA loads of one K tile and one V tile (keys row .. row+63).
template <int D>
__device__ __forceinline__ void load_kv_tile(const CUtensorMap* mk, const CUtensorMap* mv, uint8_t* sk, uint8_t* sv,
                                             uint64_t* bar, int row) {
  mbar_arrive_expect_tx(bar, 2 * AttnSmem<D>::TILE_BYTES);
#pragma unroll
  for (int h = 0; h < AttnSmem<D>::HALVES; ++h) {
    tma_load_2d(sk + h * 8192, mk, bar, h * 64, row);
    tma_load_2d(sv + h * 8192, mv, bar, h * 64, row);
  }
}

// ============================================================================ decode

// Transpose of an 8 x 8 matrix of 16-bit values held as a warp fragment (thread
// t holds row t / 4, columns 2 (t % 4), 2 (t % 4) + 1): afterwards thread t holds
// row t / 4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// NARROW (a CTA serves at most 8 query heads): S^T = K q^T with the warp's 16
// keys as the MMA rows and the heads as its 8 columns, and O^T = V^T P^T, so
// no MMA row is spent on a missing head (half the MMAs and exponentials of the
// heads-as-rows form kept for groups of 9..16 heads).
template <int D, bool NARROW>
__global__ void __launch_bounds__(160)
    attn_decode_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                       const bf16* __restrict__ q, bf16* __restrict__ o, float* __restrict__ part_o,
                       float* __restrict__ part_ml, int* __restrict__ counters, const int* __restrict__ start_pos,
                       int sp_scalar, int H, int Hkv, int S_max, int hpc, int CK, int max_chunks, int* err) {
  constexpr int STAGES = 3;
  constexpr uint32_t TB = AttnSmem<D>::TILE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + STAGES * 2 * TB);
  uint64_t* empty = full + STAGES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int n_rep = H / Hkv, groups = n_rep / hpc;
  const int chunk = blockIdx.x;
  const int z = blockIdx.y;
  const int b = z / (Hkv * groups);
  const int kvh = (z / groups) % Hkv;
  const int grp = z % groups;
  // positions are read before pdl_wait: inputs of the call, or written by a kernel that has completed (pdl_wait)
  const int sp = start_pos ? start_pos[b] : sp_scalar;
  const int L = min(sp + 1, S_max);  // keys 0 .. sp
  const int k_begin = chunk * CK;
  if (k_begin >= L) return;  // ragged batches: this sequence has fewer chunks
  const int k_end = min(L, k_begin + CK);
  const int nc = (L + CK - 1) / CK;  // chunks of this sequence
  const int n_tiles = (k_end - k_begin + KT - 1) / KT;
  const int row0 = (b * Hkv + kvh) * S_max + k_begin;
  const int h0 = kvh * n_rep + grp * hpc;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    // Cache tiles that end before this step's position were written by earlier
    // calls, which have completed (see pdl_wait): fetch up to a ring of them
    // while the QKV kernel that writes position sp is still finishing.
    const int safe = (k_end - 1 < sp) ? n_tiles : (sp - k_begin) / KT;
    const int pre = min(STAGES, safe);
    if (lane == 0) {
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      for (int j = 0; j < pre; ++j)
        load_kv_tile<D>(&map_k, &map_v, base + j * 2 * TB, base + j * 2 * TB + TB, &full[j], row0 + j * KT);
    }
    __syncwarp();
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
      int j = pre;
      for (; j < n_tiles; ++j) {
        const int st = j % STAGES;
        if (!mbar_wait(&empty[st], ((j / STAGES) & 1) ^ 1, err)) break;
        load_kv_tile<D>(&map_k, &map_v, base + st * 2 * TB, base + st * 2 * TB + TB, &full[st], row0 + j * KT);
      }
      for (int i = (j > STAGES ? j - STAGES : 0); i < j; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, err);
    }
    return;
  }
  pdl_wait();
  pdl_trigger();

  const float sl2 = rsqrtf((float)D) * LOG2E;
  __shared__ int s_abort;
  if (threadIdx.x == 0) s_abort = 0;
  asm volatile("bar.sync 1, 128;" ::: "memory");
  float* sm_o = reinterpret_cast<float*>(base);     // [4][16][D]
  float* sm_m = sm_o + 4 * 16 * D;                  // [4][16]
  float* sm_l = sm_m + 4 * 16;                      // [4][16]

  if constexpr (NARROW) {
    // ---- keys as MMA rows: thread (g, qd) holds heads 2qd, 2qd + 1 of keys g and g + 8
    const bool v0 = g < hpc;
    uint32_t qb[D / 16][2];  // B fragments of q^T: head g, d pairs 2qd (+8) of each 16-d step
    {
      const bf16* r0 = q + ((size_t)b * H + h0 + (v0 ? g : 0)) * D;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        qb[kk][0] = v0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 2 * qd) : 0u;
        qb[kk][1] = v0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 8 + 2 * qd) : 0u;
      }
    }
    float ot[D / 16][4];  // O^T: rows d = 16 i + g (+8), columns heads 2qd, 2qd + 1
#pragma unroll
    for (int i = 0; i < D / 16; ++i) ot[i][0] = ot[i][1] = ot[i][2] = ot[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2qd, 2qd + 1
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % STAGES;
      const bool ok = mbar_wait(&full[st], (j / STAGES) & 1, err);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) atomicExch(&s_abort, 1);
        break;
      }
      const int key0 = k_begin + j * KT + 16 * warp;  // first key of this warp's 16
      if (key0 < k_end) {
        const uint32_t kb = smem_u32(base + st * 2 * TB);
        const uint32_t vb = kb + TB;
        float sv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int key = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
          const int d = 16 * kk + 8 * (lane >> 4);
          uint32_t a[4];
          ldmatrix_x4(a, sw_addr(kb + (d >> 6) * 8192, key, d & 63));
          mma_bf16_16816(sv, a, qb[kk]);
        }
        sv[0] = key0 + g >= k_end ? -INFINITY : sv[0] * sl2;
        sv[1] = key0 + g >= k_end ? -INFINITY : sv[1] * sl2;
        sv[2] = key0 + g + 8 >= k_end ? -INFINITY : sv[2] * sl2;
        sv[3] = key0 + g + 8 >= k_end ? -INFINITY : sv[3] * sl2;
        float mx0 = fmaxf(sv[0], sv[2]), mx1 = fmaxf(sv[1], sv[3]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {  // over the 8 key rows g
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        // key0 < k_end: key0 itself is valid, so the maxima are finite
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float sc0 = exp2f(m0 - mn0), sc1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= sc0;
        l1 *= sc1;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          ot[c][0] *= sc0;
          ot[c][1] *= sc1;
          ot[c][2] *= sc0;
          ot[c][3] *= sc1;
        }
        sv[0] = exp2f(sv[0] - mn0);
        sv[1] = exp2f(sv[1] - mn1);
        sv[2] = exp2f(sv[2] - mn0);
        sv[3] = exp2f(sv[3] - mn1);
        l0 += sv[0] + sv[2];
        l1 += sv[1] + sv[3];
        // P^T as B fragments (key pairs 2qd (+8), head g), hi + lo bf16 parts (~16 bits of P)
        uint32_t h01, l01, h23, l23;
        split_bf16x2(sv[0], sv[1], h01, l01);
        split_bf16x2(sv[2], sv[3], h23, l23);
        const uint32_t bh[2] = {movmatrix_t(h01), movmatrix_t(h23)};
        const uint32_t bl[2] = {movmatrix_t(l01), movmatrix_t(l23)};
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          const int mi = lane >> 3;
          const int key = 16 * warp + 8 * (mi >> 1) + (lane & 7);
          const int d = 16 * c + 8 * (mi & 1);
          uint32_t a[4];
          ldmatrix_x4_trans(a, sw_addr(vb + (d >> 6) * 8192, key, d & 63));
          mma_bf16_16816(ot[c], a, bh);
          mma_bf16_16816(ot[c], a, bl);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // merge the 4 warps' states through shared memory (the ring is idle now)
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*(volatile int*)&s_abort) return;  // CTA-uniform
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      sm_o[(warp * 16 + 2 * qd) * D + 16 * c + g] = ot[c][0];
      sm_o[(warp * 16 + 2 * qd + 1) * D + 16 * c + g] = ot[c][1];
      sm_o[(warp * 16 + 2 * qd) * D + 16 * c + g + 8] = ot[c][2];
      sm_o[(warp * 16 + 2 * qd + 1) * D + 16 * c + g + 8] = ot[c][3];
    }
    if (g == 0) {
      sm_m[warp * 16 + 2 * qd] = m0;
      sm_m[warp * 16 + 2 * qd + 1] = m1;
      sm_l[warp * 16 + 2 * qd] = l0;
      sm_l[warp * 16 + 2 * qd + 1] = l1;
    }
  } else {
    // query rows: g and g + 8 are heads h0 + g, h0 + g + 8 when inside the group of hpc
    uint32_t qa[D / 16][4];
    {
      const bool v0 = g < hpc, v1 = g + 8 < hpc;
      const bf16* r0 = q + ((size_t)b * H + h0 + (v0 ? g : 0)) * D;
      const bf16* r1 = q + ((size_t)b * H + h0 + (v1 ? g + 8 : 0)) * D;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        qa[kk][0] = v0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 2 * qd) : 0u;
        qa[kk][1] = v1 ? *reinterpret_cast<const uint32_t*>(r1 + 16 * kk + 2 * qd) : 0u;
        qa[kk][2] = v0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 8 + 2 * qd) : 0u;
        qa[kk][3] = v1 ? *reinterpret_cast<const uint32_t*>(r1 + 16 * kk + 8 + 2 * qd) : 0u;
      }
    }
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % STAGES;
      const bool ok = mbar_wait(&full[st], (j / STAGES) & 1, err);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) atomicExch(&s_abort, 1);
        break;
      }
      const int key0 = k_begin + j * KT + 16 * warp;  // first key of this warp's 16
      if (key0 < k_end) {
        const uint32_t kb = smem_u32(base + st * 2 * TB);
        const uint32_t vb = kb + TB;
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int mi = lane >> 3;
          const int key = 16 * warp + 8 * (mi >> 1) + (lane & 7);
          const int d = 16 * kk + 8 * (mi & 1);
          uint32_t bf[4];
          ldmatrix_x4(bf, sw_addr(kb + (d >> 6) * 8192, key, d & 63));
          const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
          mma_bf16_16816(s[0], qa[kk], b0);
          mma_bf16_16816(s[1], qa[kk], b1);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int jn = 0; jn < 2; ++jn)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v = s[jn][e] * sl2;
            if (key0 + 8 * jn + 2 * qd + (e & 1) >= k_end) v = -INFINITY;
            s[jn][e] = v;
            if (e < 2)
              mx0 = fmaxf(mx0, v);
            else
              mx1 = fmaxf(mx1, v);
          }
        mx0 = quad_max(mx0);
        mx1 = quad_max(mx1);
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float sc0 = exp2f(m0 - mn0), sc1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= sc0;
        l1 *= sc1;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          oacc[i][0] *= sc0;
          oacc[i][1] *= sc0;
          oacc[i][2] *= sc1;
          oacc[i][3] *= sc1;
        }
#pragma unroll
        for (int jn = 0; jn < 2; ++jn) {
          s[jn][0] = exp2f(s[jn][0] - mn0);
          s[jn][1] = exp2f(s[jn][1] - mn0);
          s[jn][2] = exp2f(s[jn][2] - mn1);
          s[jn][3] = exp2f(s[jn][3] - mn1);
          l0 += s[jn][0] + s[jn][1];
          l1 += s[jn][2] + s[jn][3];
        }
        // P as a sum of two bf16 parts (hi + lo): the decode kernel is bound by
        // the cache stream, so the second MMA is free and P keeps ~16 bits.
        uint32_t ph[4], pl[4];
        split_bf16x2(s[0][0], s[0][1], ph[0], pl[0]);
        split_bf16x2(s[0][2], s[0][3], ph[1], pl[1]);
        split_bf16x2(s[1][0], s[1][1], ph[2], pl[2]);
        split_bf16x2(s[1][2], s[1][3], ph[3], pl[3]);
#pragma unroll
        for (int jd = 0; jd < D / 8; jd += 2) {
          const int mi = lane >> 3;
          const int key = 16 * warp + 8 * (mi & 1) + (lane & 7);
          const int d = 8 * (jd + (mi >> 1));
          uint32_t bf[4];
          ldmatrix_x4_trans(bf, sw_addr(vb + (d >> 6) * 8192, key, d & 63));
          const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
          mma_bf16_16816(oacc[jd], ph, b0);
          mma_bf16_16816(oacc[jd], pl, b0);
          mma_bf16_16816(oacc[jd + 1], ph, b1);
          mma_bf16_16816(oacc[jd + 1], pl, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // merge the 4 warps' states through shared memory (the ring is idle now)
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*(volatile int*)&s_abort) return;  // CTA-uniform
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      sm_o[(warp * 16 + g) * D + 8 * i + 2 * qd] = oacc[i][0];
      sm_o[(warp * 16 + g) * D + 8 * i + 2 * qd + 1] = oacc[i][1];
      sm_o[(warp * 16 + g + 8) * D + 8 * i + 2 * qd] = oacc[i][2];
      sm_o[(warp * 16 + g + 8) * D + 8 * i + 2 * qd + 1] = oacc[i][3];
    }
    if (qd == 0) {
      sm_m[warp * 16 + g] = m0;
      sm_m[warp * 16 + g + 8] = m1;
      sm_l[warp * 16 + g] = l0;
      sm_l[warp * 16 + g + 8] = l1;
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  for (int e = threadIdx.x; e < hpc * D; e += 128) {
    const int r = e / D, d = e - r * D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, sm_m[w * 16 + r]);
    float acc = 0.f, ll = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sm_m[w * 16 + r];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - mm);
      acc += sm_o[(w * 16 + r) * D + d] * f;
      ll += sm_l[w * 16 + r] * f;
    }
    if (nc == 1) {  // the sequence's only chunk: normalise and store the output directly
      o[((size_t)b * H + h0 + r) * D + d] = __float2bfloat16_rn(acc / ll);
      continue;
    }
    const size_t slot = ((size_t)b * H + h0 + r) * max_chunks + chunk;
    part_o[slot * D + d] = acc;
    if (d == 0) {
      part_ml[slot * 2] = mm;
      part_ml[slot * 2 + 1] = ll;
    }
  }
  if (nc == 1) return;

  // The CTA that finishes last for this (sequence, head group) merges every
  // chunk's partial with the log-sum-exp rule, in chunk order (deterministic),
  // and re-arms the counter for the next launch.
  asm volatile("bar.sync 1, 128;" ::: "memory");
  __shared__ int s_last;
  if (threadIdx.x == 0) s_last = (atomic_add_acq_rel(&counters[z], 1) == nc - 1);
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (!s_last) return;
  for (int e = threadIdx.x; e < hpc * D; e += 128) {
    const int r = e / D, d = e - r * D;
    const size_t row = ((size_t)b * H + h0 + r) * max_chunks;
    float mm = -INFINITY;
    for (int c = 0; c < nc; ++c) mm = fmaxf(mm, __ldcg(part_ml + (row + c) * 2));
    float acc = 0.f, ll = 0.f;
    for (int c = 0; c < nc; ++c) {
      const float f = exp2f(__ldcg(part_ml + (row + c) * 2) - mm);
      ll += __ldcg(part_ml + (row + c) * 2 + 1) * f;
      acc += __ldcg(part_o + (row + c) * D + d) * f;
    }
    o[((size_t)b * H + h0 + r) * D + d] = __float2bfloat16_rn(acc / ll);
  }
  if (threadIdx.x == 0) counters[z] = 0;
}

// ============================================================================ fp32 mode

template <typename T>
__global__ void attn_simple_kernel(const T* __restrict__ q, const T* __restrict__ ck, const T* __restrict__ cv,
                                   T* __restrict__ o, const int* __restrict__ start_pos, int sp_scalar, int T_, int H,
                                   int Hkv, int D, int S_max) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float sm[];
  float* qs = sm;             // [D]
  float* sc = sm + D;         // [S_max]
  __shared__ float red[32];
  const int t = blockIdx.x, h = blockIdx.y;
  const int b = t / T_, s = t - b * T_;
  const int pos = min((start_pos ? start_pos[b] : sp_scalar) + s, S_max - 1);
  const int kvh = h / (H / Hkv);
  const float scale = rsqrtf((float)D);
  for (int d = threadIdx.x; d < D; d += blockDim.x) qs[d] = to_f32(q[((size_t)t * H + h) * D + d]);
  __syncthreads();
  const T* K = ck + (size_t)(b * Hkv + kvh) * S_max * D;
  const T* V = cv + (size_t)(b * Hkv + kvh) * S_max * D;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j <= pos; j += blockDim.x) {
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(qs[d], to_f32(K[(size_t)j * D + d]), acc);
    sc[j] = acc * scale;
    mx = fmaxf(mx, sc[j]);
  }
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    red[0] = m;
  }
  __syncthreads();
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j <= pos; j += blockDim.x) {
    const float e = expf(sc[j] - mx);
    sc[j] = e;
    sum += e;
  }
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s2 = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s2 += red[w];
    red[0] = s2;
  }
  __syncthreads();
  const float inv = 1.f / red[0];
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j <= pos; ++j) acc = fmaf(sc[j], to_f32(V[(size_t)j * D + d]), acc);
    o[((size_t)t * H + h) * D + d] = from_f32<T>(acc * inv);
  }
}

// ============================================================================ host launchers

DecodePlan plan_decode(int B, int H, int Hkv, int S_max, int max_len, int num_sms) {
  DecodePlan p;
  const int n_rep = H / Hkv;
  p.hpc = decode_heads_per_cta(n_rep);
  const int units = B * Hkv * (n_rep / p.hpc);
  // chunks per unit so that the grid covers the SMs about twice (at least one tile each)
  int want = (2 * num_sms + units - 1) / units;
  int ck = (max_len + want - 1) / want;
  ck = (ck + KT - 1) / KT * KT;
  if (ck < 128) ck = 128;  // at least two tiles per CTA (measured: 128 beats 256 and 512 on short histories)
  if (ck > 2048) ck = 2048;  // measured: 2048 beats 1024 and 4096 on long ragged histories (8B decode)
  p.CK = ck;
  p.max_chunks = (S_max + ck - 1) / ck;
  p.part_floats = (size_t)B * H * p.max_chunks * 128 + (size_t)B * H * p.max_chunks * 2;
  return p;
}

bool check_decode_heads(int H, int Hkv, int hpc) {
  if (Hkv < 1 || H % Hkv || hpc < 1 || hpc > 16) return false;
  const int n_rep = H / Hkv, groups = n_rep / hpc;
  std::vector<int> seen(H, 0);
  for (int kvh = 0; kvh < Hkv; ++kvh)
    for (int grp = 0; grp < groups; ++grp)
      for (int r = 0; r < hpc; ++r) {  // the kernels' head index h0 + r
        const int h = kvh * n_rep + grp * hpc + r;
        if (h < 0 || h >= H || h / n_rep != kvh) return false;
        ++seen[h];
      }
  for (int v : seen)
    if (v != 1) return false;
  return true;
}

template <int D>
static cudaError_t decode_d(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                            int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int S_max,
                            const DecodePlan& p, int* err, cudaStream_t st) {
  const size_t smem = 1024 + 3 * 2 * AttnSmem<D>::TILE_BYTES + 64;
  const bool narrow = p.hpc <= 8;
  static std::atomic<unsigned long long> attr{0}, attr_n{0};
  cudaError_t e = narrow ? ensure_smem(attn_decode_kernel<D, true>, smem, attr_n)
                         : ensure_smem(attn_decode_kernel<D, false>, smem, attr);
  if (e != cudaSuccess) return e;
  const int n_rep = H / Hkv;
  float* part_o = part;
  float* part_ml = part + (size_t)B * H * p.max_chunks * D;
  dim3 grid(p.max_chunks, B * Hkv * (n_rep / p.hpc));
  return launch_pdl(narrow ? attn_decode_kernel<D, true> : attn_decode_kernel<D, false>, grid, dim3(160), smem, st,
                    mk, mv, reinterpret_cast<const bf16*>(q),
                    reinterpret_cast<bf16*>(o), part_o, part_ml, counters, sp, sp_scalar, H, Hkv, S_max, p.hpc, p.CK,
                    p.max_chunks, err);
}

cudaError_t launch_attn_decode(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                               int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int D, int S_max,
                               const DecodePlan& p, int* err, cudaStream_t st) {
  if (D == 128) return decode_d<128>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
  return decode_d<64>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
}

template <typename T>
cudaError_t launch_attn_simple(const void* q, const void* ck, const void* cv, void* o, const int* sp, int sp_scalar,
                               int B, int T_, int H, int Hkv, int D, int S_max, cudaStream_t st) {
  const size_t smem = (size_t)(D + S_max) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_simple_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(B * T_, H);
  return launch_pdl(attn_simple_kernel<T>, grid, dim3(128), smem, st, reinterpret_cast<const T*>(q),
                    reinterpret_cast<const T*>(ck), reinterpret_cast<const T*>(cv), reinterpret_cast<T*>(o), sp,
                    sp_scalar, T_, H, Hkv, D, S_max);
}

template cudaError_t launch_attn_simple<float>(const void*, const void*, const void*, void*, const int*, int, int,
                                               int, int, int, int, int, cudaStream_t);
template cudaError_t launch_attn_simple<bf16>(const void*, const void*, const void*, void*, const int*, int, int, int,
                                              int, int, int, int, cudaStream_t);

}  // namespace llama
