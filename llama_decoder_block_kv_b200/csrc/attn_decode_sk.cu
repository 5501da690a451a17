// Split-K flash-decode attention (T == 1) with the key tiles dealt out
// stream-K style: the same computation as attn_decode_kernel (attention.cu) —
// for each sequence b and query head h, softmax_j(q.k_j / sqrt(D)) over the
// cached keys j <= start_pos[b] of kv head h / n_rep, times V ("LLaMA: Open
// and Efficient Foundation Language Models" notes, Attention.forward and
// repeat_kv) — with a different split of the work.
//
// A unit is (sequence, kv head, group of hpc query heads); its history is
// n_b = ceil(L_b / 64) key tiles. The tiles of all units, unit-major, form
// one list of W tiles that is cut into equal contiguous ranges, one per CTA
// (2 per SM), so every CTA streams the same number of K/V bytes whatever the
// lengths of the sequences (no partially filled last wave). A CTA walks its
// range as segments (a run of tiles of one unit):
//   warp 4      TMA producer: the K and V tiles of the range through a
//               3-stage ring (128-byte swizzle, no multicast), crossing
//               segment edges without pausing; tiles of positions written by
//               earlier calls are fetched before griddepcontrol.wait;
//   warps 0..3  warp w takes keys 16w .. 16w + 15 of every tile on the
//               warp-level bf16 tensor-core MMA with its own online-softmax
//               state (max, sum, O over the whole head dimension); P is split
//               into two bf16 parts for the MMA (~16 bits kept). At the end of
//               a segment the four states merge in the ring stage of the
//               segment's last tile, which is released only after the merge.
// A segment that covers its whole unit writes the output; otherwise it writes
// an unnormalised partial (max, sum, O) and the CTA that arrives last for the
// unit merges the partials of its contributing CTAs in CTA order with the
// log-sum-exp rule (deterministic), then re-arms the unit's counter.
#include "kernels.cuh"

#include <algorithm>
#include <vector>

namespace llama {

namespace {
constexpr int SKT = 64;      // keys per tile
constexpr int SK_STAGES = 3;
constexpr float SK_LOG2E = 1.4426950408889634f;
}  // namespace

// element (row, col) of a 64-row x 64-column bf16 box written with 128-byte swizzling
__device__ __forceinline__ uint32_t sk_sw(uint32_t box, int row, int col) {
  return box + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2;
}
__device__ __forceinline__ float sk_quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float sk_quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// Stream-K split of W tiles over G CTAs (G <= W, W * G < 2^32, checked by the
// plan): CTA c owns [begin(c), begin(c+1)); owner(x) is the CTA whose range holds tile x.
__host__ __device__ __forceinline__ uint32_t sk_begin(uint32_t c, uint32_t W, uint32_t G) { return c * W / G; }
__host__ __device__ __forceinline__ uint32_t sk_own(uint32_t x, uint32_t W, uint32_t G) { return ((x + 1) * G - 1) / W; }

// Where tile x lies: units of sequence b occupy [pb[b] * HG, pb[b + 1] * HG), n_b tiles each.
struct SkUnit {
  int b, zl;  // sequence, unit inside the sequence (kv head * groups + group)
  int t;      // tile inside the unit
};
__host__ __device__ __forceinline__ SkUnit sk_locate(const int* pb, const int* nb, int B, int HG, uint32_t x) {
  int lo = 0, hi = B - 1;  // the last b with pb[b] * HG <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((uint32_t)pb[mid] * (uint32_t)HG <= x) lo = mid; else hi = mid - 1;
  }
  SkUnit u;
  u.b = lo;
  const uint32_t off = x - (uint32_t)pb[lo] * (uint32_t)HG;
  u.zl = (int)(off / (uint32_t)nb[lo]);
  u.t = (int)(off - (uint32_t)u.zl * (uint32_t)nb[lo]);
  return u;
}

// floats of one partial: O [hpc][D], then (max, sum) per head, padded to 16 bytes
__host__ __device__ __forceinline__ int sk_part_stride(int hpc, int D) { return hpc * D + ((2 * hpc + 3) & ~3); }

// Transpose of an 8 x 8 matrix of 16-bit values held as a warp fragment (thread
// t holds row t / 4, columns 2 (t % 4), 2 (t % 4) + 1): afterwards thread t holds
// row t / 4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// NARROW (a unit serves at most 8 query heads): the scores are computed as
// S^T = K q^T with the 16 keys of a warp as the MMA rows and the heads as its
// 8 columns, and the output as O^T = V^T P^T (head dimension as rows), so no
// MMA row is spent on a missing head: half the MMAs and exponentials of the
// heads-as-rows form, which the wider groups (9..16 heads) keep.
template <int D, bool NARROW>
__global__ void __launch_bounds__(160, 2)
    attn_decode_sk_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                          const bf16* __restrict__ q, bf16* __restrict__ o, float* __restrict__ part,
                          int* __restrict__ counters, const int* __restrict__ start_pos, int sp_scalar, int B, int H,
                          int Hkv, int S_max, int hpc, int* err) {
  constexpr uint32_t TB = SKT * D * 2;  // one K or one V tile
  constexpr int HALVES = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + SK_STAGES * 2 * TB);
  uint64_t* empty = full + SK_STAGES;
  int* nb = reinterpret_cast<int*>(empty + SK_STAGES);  // [B] tiles per unit of each sequence
  int* pb = nb + B;                                      // [B + 1] prefix sums of nb
  __shared__ float s_m[64], s_l[64];  // (max, sum) of [4 warps][16 rows] at a segment's merge
  __shared__ int s_last;
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_rep = H / Hkv, groups = n_rep / hpc, HG = Hkv * groups;
  const int pstride = sk_part_stride(hpc, D);

  // Positions are inputs of the call or written by a kernel that has completed
  // (the launch order guarantees it for every kernel before the predecessor).
  for (int b = tid; b < B; b += blockDim.x) {
    const int sp = start_pos ? start_pos[b] : sp_scalar;
    const int L = max(1, min(sp + 1, S_max));
    nb[b] = (L + SKT - 1) / SKT;
  }
  if (tid == 0) {
    for (int i = 0; i < SK_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int b = 0; b < B; ++b) {
      pb[b] = acc;
      acc += nb[b];
    }
    pb[B] = acc;
  }
  __syncthreads();
  const uint32_t W = (uint32_t)pb[B] * (uint32_t)HG;
  const uint32_t G = min((uint32_t)gridDim.x, W);
  const uint32_t cta = blockIdx.x;
  const uint32_t sbeg = cta < G ? sk_begin(cta, W, G) : 0u, send = cta < G ? sk_begin(cta + 1, W, G) : 0u;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && sbeg < send) {
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      SkUnit u = sk_locate(pb, nb, B, HG, sbeg);
      int j = 0;
      bool waited = false;
      for (uint32_t x = sbeg; x < send; ++x, ++j) {
        const int sp = start_pos ? start_pos[u.b] : sp_scalar;
        // tiles that end before this step's position were written by earlier
        // calls; the one holding the position waits for the kernel writing it
        if (!waited && (j == SK_STAGES || u.t * SKT + SKT - 1 >= sp)) {
          pdl_wait();
          pdl_trigger();
          waited = true;
        }
        const int st = j % SK_STAGES;
        if (!wait_or_abort(&empty[st], ((j / SK_STAGES) & 1) ^ 1, err, abort_flag)) break;
        const int kvh = u.zl / groups;
        const int row = (u.b * Hkv + kvh) * S_max + u.t * SKT;
        uint8_t* kd = base + st * 2 * TB;
        mbar_arrive_expect_tx(&full[st], 2 * TB);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          tma_load_2d(kd + h * 8192, &map_k, &full[st], h * 64, row);
          tma_load_2d(kd + TB + h * 8192, &map_v, &full[st], h * 64, row);
        }
        if (++u.t == nb[u.b]) {
          u.t = 0;
          if (++u.zl == HG) {
            u.zl = 0;
            ++u.b;
          }
        }
      }
      if (!waited) {
        pdl_wait();
        pdl_trigger();
      }
      // no copy may be in flight when the CTA exits
      for (int i = (j > SK_STAGES ? j - SK_STAGES : 0); i < j; ++i)
        mbar_wait(&full[i % SK_STAGES], (i / SK_STAGES) & 1, err);
    } else if (lane == 0) {
      pdl_wait();
      pdl_trigger();
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  pdl_wait();
  pdl_trigger();
  const int g = lane >> 2, qd = lane & 3;
  const float sl2 = rsqrtf((float)D) * SK_LOG2E;
  const bool rv0 = g < hpc, rv1 = g + 8 < hpc;  // rows g, g + 8 are heads of the group
  int j = 0;
  uint32_t x = sbeg;
  while (x < send) {
    const SkUnit u = sk_locate(pb, nb, B, HG, x);
    const int n_u = nb[u.b];
    const int seg_len = (int)min(send - x, (uint32_t)(n_u - u.t));
    const int z = u.b * HG + u.zl;
    const int kvh = u.zl / groups, grp = u.zl - kvh * groups;
    const int h0 = kvh * n_rep + grp * hpc;
    const int sp = start_pos ? start_pos[u.b] : sp_scalar;
    const int L = max(1, min(sp + 1, S_max));

    int st = 0;  // the ring stage of the segment's last tile
    if constexpr (NARROW) {
      // ---- keys as MMA rows: thread (g, qd) holds heads 2qd, 2qd + 1 of keys g and g + 8
      uint32_t qb[D / 16][2];  // B fragments of q^T: head g, d pairs 2qd (+8) of each 16-d step
      {
        const bf16* r0 = q + ((size_t)u.b * H + h0 + (rv0 ? g : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          qb[kk][0] = rv0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 2 * qd) : 0u;
          qb[kk][1] = rv0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 8 + 2 * qd) : 0u;
        }
      }
      float ot[D / 16][4];  // O^T: rows d = 16 i + g (+8), columns heads 2qd, 2qd + 1
#pragma unroll
      for (int i = 0; i < D / 16; ++i) ot[i][0] = ot[i][1] = ot[i][2] = ot[i][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2qd, 2qd + 1
      for (int i = 0; i < seg_len; ++i, ++j) {
        st = j % SK_STAGES;
        const bool ok = wait_or_abort(&full[st], (j / SK_STAGES) & 1, err, abort_flag);
        const int key0 = (u.t + i) * SKT + 16 * warp;  // first of this warp's 16 keys
        if (__all_sync(0xffffffffu, ok) && key0 < L) {
          const uint32_t kb = smem_u32(base + st * 2 * TB), vb = kb + TB;
          float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int key = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int d = 16 * kk + 8 * (lane >> 4);
            uint32_t a[4];
            ldmatrix_x4(a, sk_sw(kb + (d >> 6) * 8192, key, d & 63));
            mma_bf16_16816(s, a, qb[kk]);
          }
          // scale; keys at or past the history's end are masked
          s[0] = key0 + g >= L ? -INFINITY : s[0] * sl2;
          s[1] = key0 + g >= L ? -INFINITY : s[1] * sl2;
          s[2] = key0 + g + 8 >= L ? -INFINITY : s[2] * sl2;
          s[3] = key0 + g + 8 >= L ? -INFINITY : s[3] * sl2;
          float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {  // over the 8 key rows g
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          // key0 < L: key0 itself is valid, so the maxima are finite
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
          s[0] = exp2f(s[0] - mn0);
          s[1] = exp2f(s[1] - mn1);
          s[2] = exp2f(s[2] - mn0);
          s[3] = exp2f(s[3] - mn1);
          l0 += s[0] + s[2];
          l1 += s[1] + s[3];
          // P^T as B fragments (key pairs 2qd (+8), head g), hi + lo bf16 parts:
          // transpose the [key][head] fragments of keys 0-7 and 8-15
          uint32_t h01, l01, h23, l23;
          split_bf16x2(s[0], s[1], h01, l01);
          split_bf16x2(s[2], s[3], h23, l23);
          const uint32_t bh[2] = {movmatrix_trans(h01), movmatrix_trans(h23)};
          const uint32_t bl[2] = {movmatrix_trans(l01), movmatrix_trans(l23)};
          // O^T += V^T P^T over this warp's 16 keys; V^T fragments by transposed loads of V
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            const int mi = lane >> 3;
            const int key = 16 * warp + 8 * (mi >> 1) + (lane & 7);
            const int d = 16 * c + 8 * (mi & 1);
            uint32_t a[4];
            ldmatrix_x4_trans(a, sk_sw(vb + (d >> 6) * 8192, key, d & 63));
            mma_bf16_16816(ot[c], a, bh);
            mma_bf16_16816(ot[c], a, bl);
          }
        }
        if (i + 1 < seg_len) {  // the segment's last stage is released after the merge below
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[st]);
        }
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      // this warp's state -> [warp][head][D] in the stage of the segment's last tile
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float* so = reinterpret_cast<float*>(base + st * 2 * TB);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        so[(warp * 16 + 2 * qd) * D + 16 * c + g] = ot[c][0];
        so[(warp * 16 + 2 * qd + 1) * D + 16 * c + g] = ot[c][1];
        so[(warp * 16 + 2 * qd) * D + 16 * c + g + 8] = ot[c][2];
        so[(warp * 16 + 2 * qd + 1) * D + 16 * c + g + 8] = ot[c][3];
      }
      if (g == 0) {
        s_m[warp * 16 + 2 * qd] = m0;
        s_m[warp * 16 + 2 * qd + 1] = m1;
        s_l[warp * 16 + 2 * qd] = l0;
        s_l[warp * 16 + 2 * qd + 1] = l1;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    } else {
      uint32_t qa[D / 16][4];
      {
        const bf16* r0 = q + ((size_t)u.b * H + h0 + (rv0 ? g : 0)) * D;
        const bf16* r1 = q + ((size_t)u.b * H + h0 + (rv1 ? g + 8 : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          qa[kk][0] = rv0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 2 * qd) : 0u;
          qa[kk][1] = rv1 ? *reinterpret_cast<const uint32_t*>(r1 + 16 * kk + 2 * qd) : 0u;
          qa[kk][2] = rv0 ? *reinterpret_cast<const uint32_t*>(r0 + 16 * kk + 8 + 2 * qd) : 0u;
          qa[kk][3] = rv1 ? *reinterpret_cast<const uint32_t*>(r1 + 16 * kk + 8 + 2 * qd) : 0u;
        }
      }
      float oacc[D / 8][4];
#pragma unroll
      for (int c = 0; c < D / 8; ++c) oacc[c][0] = oacc[c][1] = oacc[c][2] = oacc[c][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

      for (int i = 0; i < seg_len; ++i, ++j) {
        st = j % SK_STAGES;
        const bool ok = wait_or_abort(&full[st], (j / SK_STAGES) & 1, err, abort_flag);
        const int key0 = (u.t + i) * SKT + 16 * warp;  // first of this warp's 16 keys
        if (__all_sync(0xffffffffu, ok) && key0 < L) {
          const uint32_t kb = smem_u32(base + st * 2 * TB), vb = kb + TB;
          float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int mi = lane >> 3;
            const int key = 16 * warp + 8 * (mi >> 1) + (lane & 7);
            const int d = 16 * kk + 8 * (mi & 1);
            uint32_t bf[4];
            ldmatrix_x4(bf, sk_sw(kb + (d >> 6) * 8192, key, d & 63));
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
              if (key0 + 8 * jn + 2 * qd + (e & 1) >= L) v = -INFINITY;
              s[jn][e] = v;
              if (e < 2)
                mx0 = fmaxf(mx0, v);
              else
                mx1 = fmaxf(mx1, v);
            }
          // key0 < L: the maxima are finite
          const float mn0 = fmaxf(m0, sk_quad_max(mx0)), mn1 = fmaxf(m1, sk_quad_max(mx1));
          const float sc0 = exp2f(m0 - mn0), sc1 = exp2f(m1 - mn1);
          m0 = mn0;
          m1 = mn1;
          l0 *= sc0;
          l1 *= sc1;
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            oacc[c][0] *= sc0;
            oacc[c][1] *= sc0;
            oacc[c][2] *= sc1;
            oacc[c][3] *= sc1;
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
          // O += P V over this warp's 16 keys, P as hi + lo bf16 parts
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
            ldmatrix_x4_trans(bf, sk_sw(vb + (d >> 6) * 8192, key, d & 63));
            const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
            mma_bf16_16816(oacc[jd], ph, b0);
            mma_bf16_16816(oacc[jd], pl, b0);
            mma_bf16_16816(oacc[jd + 1], ph, b1);
            mma_bf16_16816(oacc[jd + 1], pl, b1);
          }
        }
        if (i + 1 < seg_len) {  // the segment's last stage is released after the merge below
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[st]);
        }
      }
      l0 = sk_quad_sum(l0);
      l1 = sk_quad_sum(l1);
      // this warp's state -> [warp][head][D] in the stage of the segment's last tile
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float* so = reinterpret_cast<float*>(base + st * 2 * TB);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        *reinterpret_cast<float2*>(so + (warp * 16 + g) * D + 8 * c + 2 * qd) = make_float2(oacc[c][0], oacc[c][1]);
        *reinterpret_cast<float2*>(so + (warp * 16 + g + 8) * D + 8 * c + 2 * qd) =
            make_float2(oacc[c][2], oacc[c][3]);
      }
      if (qd == 0) {
        s_m[warp * 16 + g] = m0;
        s_m[warp * 16 + g + 8] = m1;
        s_l[warp * 16 + g] = l0;
        s_l[warp * 16 + g + 8] = l1;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    // Merge the four warps' states, held in the stage of the segment's last
    // tile, which every warp has finished reading: [4 warps][16 rows][D] floats
    // fill its 2 x 64 x D bf16 exactly; the (max, sum) pairs are in s_m, s_l.
    float* sm_o = reinterpret_cast<float*>(base + st * 2 * TB);
    const uint32_t P = (uint32_t)pb[u.b] * (uint32_t)HG + (uint32_t)u.zl * (uint32_t)n_u;  // the unit's first tile
    const bool whole = u.t == 0 && seg_len == n_u;
    // Partial state of this CTA for a split unit: slot 2 cta when the unit began
    // before this range (the range's first segment), else slot 2 cta + 1 (the
    // unit runs past the range's end: its last segment).
    float* pp = part + (size_t)(2 * cta + (P <= sbeg ? 0 : 1)) * pstride;
    for (int e = tid; e < hpc * D; e += 128) {
      const int r = e / D, d = e - r * D;
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) mm = fmaxf(mm, s_m[w * 16 + r]);
      float acc = 0.f, ll = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = s_m[w * 16 + r];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - mm);  // a warp without valid keys in the segment
        acc += sm_o[(w * 16 + r) * D + d] * f;
        ll += s_l[w * 16 + r] * f;
      }
      if (whole) {  // the whole unit is in this range: normalise and store
        o[((size_t)u.b * H + h0 + r) * D + d] = __float2bfloat16_rn(acc / ll);
      } else {
        __stcg(pp + r * D + d, acc);
        if (d == 0) __stcg(reinterpret_cast<float2*>(pp + hpc * D + 2 * r), make_float2(mm, ll));
      }
    }
    fence_proxy_async_smem();  // these generic writes come before the next TMA write into the stage
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (lane == 0) mbar_arrive(&empty[st]);

    if (!whole) {
      const uint32_t c0 = sk_own(P, W, G), c1 = sk_own(P + n_u - 1, W, G);
      if (tid == 0) s_last = (atomic_add_acq_rel(&counters[z], 1) == (int)(c1 - c0));
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (s_last) {
        // The last contributor merges the partials of CTAs c0 .. c1 in that
        // order: m = max m_c, l = sum l_c 2^(m_c - m), o = sum o_c 2^(m_c - m) / l.
        // CTA c0 holds the unit in its second slot unless its range starts at
        // the unit; every later contributor holds it in its first slot.
        const uint32_t slot0 = 2 * c0 + (sk_begin(c0, W, G) == P ? 0u : 1u);
        for (int e = tid; e < hpc * D / 4; e += 128) {
          const int r = (4 * e) / D, d = 4 * e - r * D;
          float mm = -INFINITY;
          for (uint32_t c = c0; c <= c1; ++c) {
            const float* pc = part + (size_t)(c == c0 ? slot0 : 2 * c) * pstride;
            mm = fmaxf(mm, __ldcg(pc + hpc * D + 2 * r));
          }
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          float ll = 0.f;
          for (uint32_t c = c0; c <= c1; ++c) {
            const float* pc = part + (size_t)(c == c0 ? slot0 : 2 * c) * pstride;
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(pc + hpc * D + 2 * r));
            const float f = exp2f(ml.x - mm);
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pc + r * D + d));
            ll += ml.y * f;
            acc.x += v.x * f;
            acc.y += v.y * f;
            acc.z += v.z * f;
            acc.w += v.w * f;
          }
          const float il = 1.f / ll;
          uint2 w;
          w.x = pack_bf16x2(acc.x * il, acc.y * il);
          w.y = pack_bf16x2(acc.z * il, acc.w * il);
          *reinterpret_cast<uint2*>(o + ((size_t)u.b * H + h0 + r) * D + d) = w;
        }
        if (tid == 0) counters[z] = 0;  // re-armed for the next launch
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // s_last is rewritten by the next segment
    }
    x += seg_len;
  }
}

// ------------------------------------------------------------------ host side

DecodeSkPlan plan_decode_sk(int B, int H, int Hkv, int D, int max_len, int num_sms) {
  DecodeSkPlan p;
  const int n_rep = H / Hkv;
  p.hpc = decode_heads_per_cta(n_rep);
  const long long HG = (long long)Hkv * (n_rep / p.hpc);
  const long long W_max = (long long)B * HG * ((max_len + SKT - 1) / SKT);
  // two resident CTAs per SM; at least two tiles per CTA on short histories
  const long long G = std::min<long long>(2LL * num_sms, std::max<long long>(1, W_max / 2));
  p.grid = (int)G;
  p.units = (int)(B * HG);
  p.part_floats = (size_t)2 * p.grid * sk_part_stride(p.hpc, D);
  p.ok = B >= 1 && B <= 1024 && (D == 64 || D == 128) && W_max * G < (1LL << 32) && n_rep % p.hpc == 0;
  return p;
}

// One position for the whole batch: every unit has the same number of key
// tiles, so a grid of a whole number of CTAs per unit (where that keeps at
// least 85 % of the two-per-SM slots) puts each CTA's range inside one unit.
// Measured on B200, the 70B layer at batch 16 x 4096: 0.3318 -> 0.3292 ms per
// step (256 CTAs instead of 296). Only ever shrinks the grid, so the
// workspace sized for plan_decode_sk's grid still holds the partials.
void align_decode_sk_uniform(DecodeSkPlan& p, int len, int num_sms) {
  if (!p.ok) return;
  const int cap = 2 * num_sms, n_t = (len + SKT - 1) / SKT;
  if (p.units > cap) return;
  const int cc = cap / p.units;
  if (p.units * cc * 100 >= cap * 85 && n_t >= cc && p.units * cc < p.grid) p.grid = p.units * cc;
}

static size_t sk_smem(int D, int B) {
  return 1024 + (size_t)SK_STAGES * 2 * SKT * D * 2 + 2 * SK_STAGES * 8 + (size_t)(2 * B + 1) * 4;
}

template <int D, bool NARROW>
static cudaError_t decode_sk_d(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                               int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int S_max,
                               const DecodeSkPlan& p, int* err, cudaStream_t st) {
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(attn_decode_sk_kernel<D, NARROW>, sk_smem(D, 1024), attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_decode_sk_kernel<D, NARROW>, dim3(p.grid), dim3(160), sk_smem(D, B), st, mk, mv,
                    reinterpret_cast<const bf16*>(q), reinterpret_cast<bf16*>(o), part, counters, sp, sp_scalar, B,
                    H, Hkv, S_max, p.hpc, err);
}

cudaError_t launch_attn_decode_sk(const CUtensorMap& mk, const CUtensorMap& mv, const void* q, void* o, float* part,
                                  int* counters, const int* sp, int sp_scalar, int B, int H, int Hkv, int D, int S_max,
                                  const DecodeSkPlan& p, int* err, cudaStream_t st) {
  if (!p.ok) return cudaErrorInvalidValue;
  if (p.hpc <= 8) {
    if (D == 128) return decode_sk_d<128, true>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
    return decode_sk_d<64, true>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
  }
  if (D == 128) return decode_sk_d<128, false>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
  return decode_sk_d<64, false>(mk, mv, q, o, part, counters, sp, sp_scalar, B, H, Hkv, S_max, p, err, st);
}

// Host walk of the split for the given positions, with the kernel's own
// functions: every tile in exactly one CTA's range, every unit split over
// CTAs c0..c1 with one partial from each, in the slot the merge reads, and
// no slot used twice or outside the plan's workspace.
bool check_decode_sk(const DecodeSkPlan& p, const int* start_pos, int B, int H, int Hkv, int D, int S_max) {
  if (!p.ok) return true;  // the kernel is not used for this shape
  if (!check_decode_heads(H, Hkv, p.hpc)) return false;
  const int n_rep = H / Hkv, HG = Hkv * (n_rep / p.hpc);
  std::vector<int> nb(B), pb(B + 1);
  int acc = 0;
  for (int b = 0; b < B; ++b) {
    const int L = std::max(1, std::min(start_pos[b] + 1, S_max));
    nb[b] = (L + SKT - 1) / SKT;
    pb[b] = acc;
    acc += nb[b];
  }
  pb[B] = acc;
  const uint32_t W = (uint32_t)acc * (uint32_t)HG;
  if ((unsigned long long)W * (unsigned long long)p.grid >= (1ULL << 32)) return false;
  const uint32_t G = std::min<uint32_t>((uint32_t)p.grid, W);
  const size_t pstride = sk_part_stride(p.hpc, D);
  std::vector<int> seen(W, 0);
  std::vector<std::vector<uint32_t>> slots(B * HG);
  std::vector<int> slot_use(2 * G, 0);
  for (uint32_t c = 0; c < G; ++c) {
    const uint32_t s0 = sk_begin(c, W, G), s1 = sk_begin(c + 1, W, G);
    if (s1 <= s0) return false;
    for (uint32_t x = s0; x < s1;) {
      const SkUnit u = sk_locate(pb.data(), nb.data(), B, HG, x);
      if (u.b < 0 || u.b >= B || u.zl < 0 || u.zl >= HG || u.t < 0 || u.t >= nb[u.b]) return false;
      const int seg = (int)std::min<uint32_t>(s1 - x, (uint32_t)(nb[u.b] - u.t));
      for (uint32_t y = x; y < x + seg; ++y) ++seen[y];
      const uint32_t P = (uint32_t)pb[u.b] * HG + (uint32_t)u.zl * nb[u.b];
      if (P + u.t != x) return false;
      if (!(u.t == 0 && seg == nb[u.b])) {
        const uint32_t slot = 2 * c + (P <= s0 ? 0 : 1);
        if (slot % 2 == 1 && x + seg != s1) return false;  // the second slot is the range's last segment
        if (slot % 2 == 0 && x != s0) return false;        // the first slot is its first segment
        if (++slot_use[slot] != 1) return false;
        if ((slot + 1) * pstride > p.part_floats) return false;
        slots[u.b * HG + u.zl].push_back(slot);
      }
      x += seg;
    }
  }
  for (int v : seen)
    if (v != 1) return false;
  for (int z = 0; z < B * HG; ++z) {
    if (slots[z].empty()) continue;
    const int b = z / HG, zl = z % HG;
    const uint32_t P = (uint32_t)pb[b] * HG + (uint32_t)zl * nb[b];
    const uint32_t c0 = sk_own(P, W, G), c1 = sk_own(P + nb[b] - 1, W, G);
    if (slots[z].size() != c1 - c0 + 1) return false;
    const uint32_t slot0 = 2 * c0 + (sk_begin(c0, W, G) == P ? 0u : 1u);
    for (uint32_t c = c0; c <= c1; ++c) {
      const uint32_t want = c == c0 ? slot0 : 2 * c;
      if (std::find(slots[z].begin(), slots[z].end(), want) == slots[z].end()) return false;
    }
  }
  return true;
}

}  // namespace llama
