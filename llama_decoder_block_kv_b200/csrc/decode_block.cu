// One decode step (T = 1, up to 32 sequences, bf16) of one decoder block in a
// single persistent launch: the whole of TransformerBlock.forward from the
// notes ("LLaMA: Open and Efficient Foundation Language Models" notes,
// TransformerBlock.forward and Attention.forward), with the KV-cache append.
//
// At decode time the block reads every weight byte once and does little else
// (the KV-cache section of "LLaMa-1/2/3 原理+源码——拆解": with the cache the
// bottleneck becomes memory access), so the launch is organised around one
// continuous weight stream. Each CTA (one per SM, 160 threads) has
//   warp 4      the producer: it streams this CTA's share of all four weight
//               matrices (wqkv, wo, w1|w3, w2, in that order) through a ring of
//               128-row x 64-k tiles with TMA (128-byte swizzle, no multicast),
//               never waiting for the activations: while the consumers are in
//               the attention phase or at a grid barrier, it already fills the
//               ring with the next matrix's tiles;
//   warps 0..3  the consumers, which walk the phases separated by grid-wide
//               barriers:
//     0. sums of squares of h per 128-column block (RMSNorm statistics);
//     1. h -> RMSNorm -> x (built in shared memory, the norm fused into the
//        load), x * Wqkv^T with RoPE, q store and the cache-slot append;
//     2. split-K flash-decode attention over the cache (q, K, V -> o);
//     3. o * Wo^T + h -> h, with the new row-block sums of squares;
//     4. RMSNorm(h) * W13^T -> silu(a) * b -> g;
//     5. g * W2^T + h -> h.
// The linears are stream-K over 128 x 64 weight stages like the decode GEMV
// (gemv.cu), with the k range cut into slices so that a CTA needs only its
// slice of x in shared memory; partial tiles of a row block are summed in a
// fixed order by the CTA that arrives last. Data written in one phase and read
// in a later one (h, q, o, g, the cache slot, partials, statistics) is read
// through L2 (ld.global.cg / cp.async.cg), after the grid barrier that orders it.
//
// The grid barriers need every CTA resident at once: the launch has one CTA
// per SM and each CTA takes most of an SM's shared memory, so no two share an
// SM, and the CTAs of an earlier kernel on the stream never wait for this one.
// Every wait (ring barriers, grid barriers) is bounded: past the limit it
// records LLAMA_DEV_TIMEOUT and the CTA unwinds.
#include "kernels.cuh"

#include <algorithm>
#include <vector>

namespace llama {

namespace {
constexpr int RPC = 128;                    // weight rows per stage
constexpr int KB = 64;                      // k per stage (one 128-byte swizzle row)
constexpr uint32_t W_BYTES = RPC * KB * 2;  // 16 KB
constexpr int OS = RPC + 4;                 // row stride of the fp32 output staging tile
constexpr int STAGES = DB_RING_STAGES;
constexpr int AKT = 64;                     // keys per attention tile
constexpr int AD = 128;                     // head dim of this kernel
constexpr float LOG2E_DB = 1.4426950408889634f;
}  // namespace

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ void bar_consumers() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// swizzled byte address of (row, col) in a tile of 128-byte rows written by TMA
__device__ __forceinline__ uint32_t db_sw128(uint32_t base, int row, int col) {
  return base + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4);
}
// element (row, col) of a 64-row x 64-column bf16 box with 128-byte swizzling
__device__ __forceinline__ uint32_t db_sw_elem(uint32_t box, int row, int col) {
  return box + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ float db_quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float db_quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// Stream-K split of `total` stages over `grid` CTAs: CTA c owns [begin(c),
// begin(c+1)), begin(c) = floor(c * total / grid). All products stay below
// 2^31 (the host checks total * grid). owner(x), the CTA whose range holds
// stage x, is the largest c with begin(c) <= x: floor(((x + 1) grid - 1) / total).
__host__ __device__ __forceinline__ int db_begin(int c, int total, int grid) {
  return (int)((unsigned)c * (unsigned)total / (unsigned)grid);
}
__host__ __device__ __forceinline__ int db_owner(int x, int total, int grid) {
  return (int)(((unsigned)(x + 1) * (unsigned)grid - 1u) / (unsigned)total);
}

// CTAs that take part in a linear: all of them, or one per stage when the
// linear has fewer stages than the grid has CTAs (every range non-empty).
__host__ __device__ __forceinline__ int db_grid(const DbLinear& L, int grid) { return L.total < grid ? L.total : grid; }
__host__ __device__ __forceinline__ void db_range(const DbLinear& L, int cta, int grid, int& sbeg, int& send) {
  const int gl = db_grid(L, grid);
  sbeg = cta < gl ? db_begin(cta, L.total, gl) : 0;
  send = cta < gl ? db_begin(cta + 1, L.total, gl) : 0;
}

// Stage order of a linear: slice-major, then row block, then k within the
// slice. Slice s covers k stages [s*NK/S, (s+1)*NK/S).
struct DbStage {
  int s, rb, start, len, reg_beg;  // slice, row block, first k stage and k stages of the slice, region start
};
__host__ __device__ __forceinline__ int db_slice_start(const DbLinear& L, int s) {
  return (int)((unsigned)s * (unsigned)L.NK / (unsigned)L.S);
}
__host__ __device__ __forceinline__ DbStage db_locate(const DbLinear& L, int x) {
  // slice s holds stages [RB * start(s), RB * start(s+1)): the largest s with RB * floor(s NK / S) <= x
  int s = (int)(((unsigned)(x / L.RB + 1) * (unsigned)L.S - 1u) / (unsigned)L.NK);
  if (s >= L.S) s = L.S - 1;
  while (s > 0 && L.RB * db_slice_start(L, s) > x) --s;
  while (s + 1 < L.S && L.RB * db_slice_start(L, s + 1) <= x) ++s;
  DbStage r;
  r.s = s;
  r.start = db_slice_start(L, s);
  r.len = db_slice_start(L, s + 1) - r.start;
  const int off = x - L.RB * r.start;
  r.rb = off / r.len;
  r.reg_beg = L.RB * r.start + r.rb * r.len;
  return r;
}

// Number of partial tiles of row block rb, and the slot of (slice s, CTA c).
__host__ __device__ __forceinline__ int db_contributors(const DbLinear& L, int rb, int grid, int s, int cta,
                                                        int* slot) {
  grid = db_grid(L, grid);
  int count = 0, sl = 0;
  for (int s2 = 0; s2 < L.S; ++s2) {
    const int st = db_slice_start(L, s2), ln = db_slice_start(L, s2 + 1) - st;
    const int beg = L.RB * st + rb * ln;
    const int c0 = db_owner(beg, L.total, grid), c1 = db_owner(beg + ln - 1, L.total, grid);
    if (s2 < s) sl += c1 - c0 + 1;
    if (s2 == s) sl += cta - c0;
    count += c1 - c0 + 1;
  }
  if (slot) *slot = sl;
  return count;
}

// Grid-wide barrier of the consumer threads. gbar[0] counts arrivals and only
// ever grows: every barrier takes exactly `grid` arrivals, so the arrival that
// returns v belongs to barrier number k = v / grid + 1, and the arrival that
// makes the count k * grid (the last one) publishes k in gbar[16], a separate
// 128-byte line that the other CTAs poll. Nothing is re-armed between barriers
// or launches (a timed-out wait leaves the count misaligned; the host clears
// both words when it reads the timeout flag).
// arrival on a counter: releases this CTA's earlier writes (all threads'
// writes ordered before it by a bar.sync) and acquires the writes released by
// the arrivals before it
__device__ __forceinline__ int atom_add_acq_rel_gpu_s32(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long atom_add_acq_rel_gpu(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void db_grid_sync(unsigned long long* gbar, int grid, int* err, volatile int* abort_flag) {
  bar_consumers();
  if (threadIdx.x == 0 && !*abort_flag) {
    const unsigned long long G = (unsigned long long)grid;
    const unsigned long long v = atom_add_acq_rel_gpu(gbar, 1ull);
    const unsigned long long k = v / G + 1ull;
    if (v + 1ull == k * G) {
      st_release_gpu_u64(gbar + 16, k);
    } else {
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_gpu_u64(gbar + 16) < k) {
        if (global_timer_ns() - t0 > LLAMA_WAIT_LIMIT_NS) {
          atomicOr(err, LLAMA_DEV_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
    }
  }
  bar_consumers();
}

// One attention work unit (sequence, kv head, group of query heads, chunk of
// keys), as both roles of the CTA enumerate them.
struct DbUnit {
  int z, chunk, b, kvh, grp, sp, L, k_begin, k_end, nc, n_tiles;
  size_t row0;  // first key row of the chunk in the cache [B_max][Hkv][S_max]
};
__device__ __forceinline__ bool db_unit(const DecodeBlockParams& p, int u, DbUnit& w) {
  const int groups = (p.H / p.Hkv) / p.hpc;
  w.z = u / p.max_chunks;
  w.chunk = u - w.z * p.max_chunks;
  w.b = w.z / (p.Hkv * groups);
  w.kvh = (w.z / groups) % p.Hkv;
  w.grp = w.z % groups;
  // positions: inputs of the call, or written by a kernel that has completed (read after pdl_wait)
  w.sp = p.start_pos ? p.start_pos[w.b] : p.sp_scalar;
  w.L = min(w.sp + 1, p.S_max);
  w.k_begin = w.chunk * p.CK;
  if (w.k_begin >= w.L) return false;  // a shorter sequence of a ragged batch
  w.k_end = min(w.L, w.k_begin + p.CK);
  w.nc = (w.L + p.CK - 1) / p.CK;
  w.n_tiles = (w.k_end - w.k_begin + AKT - 1) / AKT;
  w.row0 = (size_t)(w.b * p.Hkv + w.kvh) * p.S_max + w.k_begin;
  return true;
}

__device__ __forceinline__ void st_release_cta_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.s32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
// orders this thread's earlier (acquired) view of global memory before its later async-proxy (TMA) reads
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// ------------------------------------------------------------------ phases

// Phase 0: per-row-block sums of squares of h (the RMSNorm statistics).
__device__ void db_sumsq_phase(const DecodeBlockParams& p, int cta, int grid) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rbs = p.dim / RPC;
  for (int rb = cta; rb < rbs; rb += grid)
    for (int m = warp; m < p.M; m += 4) {
      const float4 a = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)m * p.dim + rb * RPC + lane * 4));
      float s = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) p.ssq[rb * p.M + m] = s;
    }
}

// x slice [M][k0, k0 + klen) of linear li into shared memory (rows padded by
// 16 bytes so that the fragment loads of 8 rows hit 8 different bank groups).
// For wqkv and w13 the slice is RMSNorm(h): bf16(bf16(h * r) * w), with
// r = rsqrt(sum of squares / dim + eps), as rmsnorm_kernel computes it.
// Returns the padded row length in elements.
__device__ int db_load_x(const DecodeBlockParams& p, int li, int k0, int klen, uint8_t* area, float* s_r) {
  const int tid = threadIdx.x, M = p.M;
  const int ksp = klen + 8, per_row = klen / 8;
  bf16* xs = reinterpret_cast<bf16*>(area);
  if (li == 0 || li == 2) {
    if (p.norm_local) {
      // the slice is the whole row: its sums of squares, one warp per row
      const int warp = tid >> 5, lane = tid & 31;
      for (int m = warp; m < M; m += 4) {
        const float* hr = p.h + (size_t)m * p.dim;
        float ss = 0.f;
        for (int i = lane * 4; i < p.dim; i += 128) {
          const float4 a = __ldcg(reinterpret_cast<const float4*>(hr + i));
          ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) s_r[m] = rsqrtf(ss / (float)p.dim + p.eps);
      }
    } else if (tid < M) {
      float ss = 0.f;
      for (int rb = 0; rb < p.dim / RPC; ++rb) ss += __ldcg(p.ssq + rb * M + tid);
      s_r[tid] = rsqrtf(ss / (float)p.dim + p.eps);
    }
    bar_consumers();
    const bf16* w = li == 0 ? p.attn_norm : p.ffn_norm;
    for (int idx = tid; idx < M * per_row; idx += 128) {
      const int m = idx / per_row, c8 = idx - m * per_row;
      const int k = k0 + c8 * 8;
      const float* hp = p.h + (size_t)m * p.dim + k;
      const float4 a = __ldcg(reinterpret_cast<const float4*>(hp));
      const float4 b = __ldcg(reinterpret_cast<const float4*>(hp + 4));
      const uint4 wu = *reinterpret_cast<const uint4*>(w + k);
      const float r = s_r[m];
      const float hv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      const float2 w0 = unpack_bf16x2(wu.x), w1 = unpack_bf16x2(wu.y), w2 = unpack_bf16x2(wu.z),
                   w3 = unpack_bf16x2(wu.w);
      const float wv[8] = {w0.x, w0.y, w1.x, w1.y, w2.x, w2.y, w3.x, w3.y};
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = round_to<bf16>(hv[e] * r) * wv[e];
      store8(xs + (size_t)m * ksp + c8 * 8, v);
    }
  } else {
    const bf16* src = li == 1 ? p.o : p.g;
    const int ld = li == 1 ? p.H * p.D : p.F;
    for (int idx = tid; idx < M * per_row; idx += 128) {
      const int m = idx / per_row, c8 = idx - m * per_row;
      const uint4 u = __ldcg(reinterpret_cast<const uint4*>(src + (size_t)m * ld + k0 + c8 * 8));
      *reinterpret_cast<uint4*>(xs + (size_t)m * ksp + c8 * 8) = u;
    }
  }
  return ksp;
}

// The epilogue of a finished row block: value chunks of 8 columns come from
// `get(m, jc, v)`; wqkv -> RoPE/q/cache, w13 -> SwiGLU (epilogue8), wo/w2 ->
// residual add into h plus the row block's sums of squares of the new h.
template <typename Get>
__device__ __forceinline__ void db_rowblock_epilogue(const DecodeBlockParams& p, int li, int rb, const EpiParams& ep,
                                                     Get get) {
  const int tid = threadIdx.x, M = p.M;
  const bool residual = li == 1 || li == 3;
  const int iters = (M * (RPC / 8) + 127) / 128;
  for (int it = 0; it < iters; ++it) {
    const int c = it * 128 + tid;
    const bool act = c < M * (RPC / 8);
    const int m = c / (RPC / 8), jc = c % (RPC / 8);
    const int n = rb * RPC + jc * 8;
    float sq = 0.f;
    if (act) {
      float v[8];
      float* hp = p.h + (size_t)m * p.dim + n;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (residual) {
        a = __ldcg(reinterpret_cast<const float4*>(hp));
        b = __ldcg(reinterpret_cast<const float4*>(hp + 4));
      }
      get(m, jc, v);
      if (residual) {
        v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
        v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
        __stcg(reinterpret_cast<float4*>(hp), make_float4(v[0], v[1], v[2], v[3]));
        __stcg(reinterpret_cast<float4*>(hp + 4), make_float4(v[4], v[5], v[6], v[7]));
#pragma unroll
        for (int e = 0; e < 8; ++e) sq += v[e] * v[e];
      } else {
        epilogue8<bf16>(ep, m, n, v);
      }
    }
    if (residual) {
      // the 16 chunks of one row are 16 consecutive threads (a half warp)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (act && jc == 0) p.ssq[rb * M + m] = sq;
    }
  }
}

// Phases 1, 3, 4, 5: this CTA's stream-K share of linear li. `j` counts ring
// stages across the whole launch, in the producer's order.
template <int MB>
__device__ void db_linear_phase(const DecodeBlockParams& p, int li, int cta, int grid, int& j, uint8_t* ring,
                                uint8_t* area, float* os, uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                int* s_last, float* s_r) {
  const DbLinear& L = p.lin[li];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int M = p.M;
  EpiParams ep;
  memset(&ep, 0, sizeof(ep));
  ep.M = M;
  ep.N = L.N;
  ep.err = p.err;
  if (li == 0) {
    ep.kind = EPI_QKV_ROPE;
    ep.q_out = p.q;
    ep.cache_k = p.cache_k;
    ep.cache_v = p.cache_v;
    ep.rope = p.rope;
    ep.start_pos = p.start_pos;
    ep.start_pos_scalar = p.sp_scalar;
    ep.T = 1;
    ep.H = p.H;
    ep.Hkv = p.Hkv;
    ep.D = p.D;
    ep.S_max = p.S_max;
  } else {
    ep.kind = EPI_SWIGLU;
    ep.g_out = p.g;
  }
  int sbeg, send;
  db_range(L, cta, grid, sbeg, send);
  const int a_row = warp * 32 + (lane & 7) + 8 * ((lane >> 3) & 1);  // + 16 t
  const int a_col = 8 * (lane >> 4);                                 // + 16 kk
  const uint32_t xbase = smem_u32(area);
  int cur_s = -1, ksp = 0;
  int x = sbeg;
  while (x < send) {
    const DbStage S = db_locate(L, x);
    const int seg_beg = x, seg_end = min(send, S.reg_beg + S.len);
    if (S.s != cur_s) {
      bar_consumers();  // every warp is done with the previous slice
      ksp = db_load_x(p, li, S.start * KB, S.len * KB, area, s_r);
      bar_consumers();
      cur_s = S.s;
    }
    float acc[2][MB][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) acc[t][mb][0] = acc[t][mb][1] = acc[t][mb][2] = acc[t][mb][3] = 0.f;

    for (; x < seg_end; ++x, ++j) {
      const int st = j % STAGES;
      const bool ok = wait_or_abort(&full[st], (j / STAGES) & 1, p.err, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        const uint32_t wb = smem_u32(ring + st * W_BYTES);
        const int k0 = (x - S.reg_beg) * KB;  // k offset inside the slice
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t bfr[MB][2];
#pragma unroll
          for (int mb = 0; mb < MB; ++mb) {
            const int m = mb * 8 + g;
            if (m < M) {
              const uint32_t addr = xbase + (uint32_t)((m * ksp + k0 + kk * 16 + 2 * q) * 2);
              bfr[mb][0] = lds32(addr);
              bfr[mb][1] = lds32(addr + 16);
            } else {
              bfr[mb][0] = bfr[mb][1] = 0u;
            }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            uint32_t a[4];
            ldmatrix_x4(a, db_sw128(wb, a_row + 16 * t, a_col + 16 * kk));
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) mma_bf16_16816(acc[t][mb], a, bfr[mb]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // fragments (row g / g+8 of each 16-row tile, tokens 2q, 2q+1) -> os[token][row]
    bar_consumers();
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
    bar_consumers();

    const int rb = S.rb, nbase = rb * RPC;
    if (L.S == 1 && seg_beg == S.reg_beg && seg_end == S.reg_beg + S.len) {
      // the whole row block in this CTA: epilogue straight from shared memory
      db_rowblock_epilogue(p, li, rb, ep, [&](int m, int jc, float* v) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = os[m * OS + jc * 8 + e];
      });
      bar_consumers();  // os is rewritten by the next segment
      continue;
    }
    int slot = 0;
    const int count = db_contributors(L, rb, grid, S.s, cta, &slot);
    for (int e = tid; e < M * (RPC / 4); e += 128) {
      const int m = e / (RPC / 4), jc = e - m * (RPC / 4);
      const float4 v = make_float4(os[m * OS + jc * 4], os[m * OS + jc * 4 + 1], os[m * OS + jc * 4 + 2],
                                   os[m * OS + jc * 4 + 3]);
      __stcg(reinterpret_cast<float4*>(p.part + ((size_t)slot * M + m) * L.N + nbase + jc * 4), v);
    }
    bar_consumers();
    if (tid == 0) *s_last = (atom_add_acq_rel_gpu_s32(&p.counters[rb], 1) == count - 1);
    bar_consumers();
    if (!*s_last) continue;
    db_rowblock_epilogue(p, li, rb, ep, [&](int m, int jc, float* v) {
      const int n = nbase + jc * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll 4
      for (int sl = 0; sl < count; ++sl) {
        const float4* src = reinterpret_cast<const float4*>(p.part + ((size_t)sl * M + m) * L.N + n);
        const float4 a = __ldcg(src), b = __ldcg(src + 1);
        v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
        v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
      }
    });
    if (tid == 0) p.counters[rb] = 0;
  }
}

// Phase 2: split-K flash decode, the same arithmetic as attn_decode_kernel
// (attention.cu): a work unit is (sequence, kv head, group of hpc query heads,
// chunk of CK keys); its 64-key K and V tiles come into shared memory with
// cp.async (double buffered, rows past the sequence filled with zeros), the 4
// warps take 16 keys of each tile, their states merge in shared memory, and
// the unit that finishes last for a (sequence, head group) merges the chunks'
// partials with the log-sum-exp rule in chunk order.
__device__ void db_attention_phase(const DecodeBlockParams& p, int cta, int grid, int& j, uint8_t* ring, uint8_t* area,
                                   uint64_t* full, uint64_t* empty, volatile int* abort_flag, int* s_last) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int n_rep = p.H / p.Hkv, hpc = p.hpc;
  const int units = p.M * p.Hkv * (n_rep / hpc) * p.max_chunks;
  const float sl2 = rsqrtf((float)AD) * LOG2E_DB;
  float* part_o = p.part;
  float* part_ml = p.part + (size_t)p.M * p.H * p.max_chunks * AD;

  for (int u = cta; u < units; u += grid) {
    DbUnit w;
    if (!db_unit(p, u, w)) continue;  // CTA-uniform
    const int b = w.b, chunk = w.chunk, z = w.z, k_begin = w.k_begin, k_end = w.k_end, nc = w.nc;
    const int n_tiles = w.n_tiles;
    const int h0 = w.kvh * n_rep + w.grp * hpc;

    // query rows g and g + 8: heads h0 + g, h0 + g + 8 when inside the group
    uint32_t qa[AD / 16][4];
    {
      const bool v0 = g < hpc, v1 = g + 8 < hpc;
      const bf16* r0 = p.q + ((size_t)b * p.H + h0 + (v0 ? g : 0)) * AD;
      const bf16* r1 = p.q + ((size_t)b * p.H + h0 + (v1 ? g + 8 : 0)) * AD;
#pragma unroll
      for (int kk = 0; kk < AD / 16; ++kk) {
        qa[kk][0] = v0 ? __ldcg(reinterpret_cast<const unsigned*>(r0 + 16 * kk + 2 * qd)) : 0u;
        qa[kk][1] = v1 ? __ldcg(reinterpret_cast<const unsigned*>(r1 + 16 * kk + 2 * qd)) : 0u;
        qa[kk][2] = v0 ? __ldcg(reinterpret_cast<const unsigned*>(r0 + 16 * kk + 8 + 2 * qd)) : 0u;
        qa[kk][3] = v1 ? __ldcg(reinterpret_cast<const unsigned*>(r1 + 16 * kk + 8 + 2 * qd)) : 0u;
      }
    }
    float oacc[AD / 8][4];
#pragma unroll
    for (int i = 0; i < AD / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int jt = 0; jt < n_tiles; ++jt, j += 2) {
      // the K tile then the V tile of keys k_begin + 64 jt .., two ring stages
      const int stk = j % STAGES, stv = (j + 1) % STAGES;
      const bool okk = wait_or_abort(&full[stk], (j / STAGES) & 1, p.err, abort_flag);
      const bool okv = wait_or_abort(&full[stv], ((j + 1) / STAGES) & 1, p.err, abort_flag);
      const int key0 = k_begin + jt * AKT + 16 * warp;  // first key of this warp's 16
      if (__all_sync(0xffffffffu, okk && okv) && key0 < k_end) {
        const uint32_t kb = smem_u32(ring + stk * W_BYTES);
        const uint32_t vb = smem_u32(ring + stv * W_BYTES);
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < AD / 16; ++kk) {
          const int mi = lane >> 3;
          const int key = 16 * warp + 8 * (mi >> 1) + (lane & 7);
          const int d = 16 * kk + 8 * (mi & 1);
          uint32_t bf[4];
          ldmatrix_x4(bf, db_sw_elem(kb + (d >> 6) * 8192, key, d & 63));
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
        mx0 = db_quad_max(mx0);
        mx1 = db_quad_max(mx1);
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float sc0 = exp2f(m0 - mn0), sc1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= sc0;
        l1 *= sc1;
#pragma unroll
        for (int i = 0; i < AD / 8; ++i) {
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
        // P as hi + lo bf16 parts, as in the decode kernel: P keeps ~16 bits
        uint32_t ph[4], pl[4];
        split_bf16x2(s[0][0], s[0][1], ph[0], pl[0]);
        split_bf16x2(s[0][2], s[0][3], ph[1], pl[1]);
        split_bf16x2(s[1][0], s[1][1], ph[2], pl[2]);
        split_bf16x2(s[1][2], s[1][3], ph[3], pl[3]);
#pragma unroll
        for (int jd = 0; jd < AD / 8; jd += 2) {
          const int mi = lane >> 3;
          const int key = 16 * warp + 8 * (mi & 1) + (lane & 7);
          const int d = 8 * (jd + (mi >> 1));
          uint32_t bf[4];
          ldmatrix_x4_trans(bf, db_sw_elem(vb + (d >> 6) * 8192, key, d & 63));
          const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
          mma_bf16_16816(oacc[jd], ph, b0);
          mma_bf16_16816(oacc[jd], pl, b0);
          mma_bf16_16816(oacc[jd + 1], ph, b1);
          mma_bf16_16816(oacc[jd + 1], pl, b1);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[stk]);
        mbar_arrive(&empty[stv]);
      }
    }

    // merge the 4 warps' states through shared memory
    bar_consumers();  // the previous unit's merge has finished reading the area
    l0 = db_quad_sum(l0);
    l1 = db_quad_sum(l1);
    float* sm_o = reinterpret_cast<float*>(area);  // [4][16][AD]
    float* sm_m = sm_o + 4 * 16 * AD;               // [4][16]
    float* sm_l = sm_m + 4 * 16;                    // [4][16]
#pragma unroll
    for (int i = 0; i < AD / 8; ++i) {
      sm_o[(warp * 16 + g) * AD + 8 * i + 2 * qd] = oacc[i][0];
      sm_o[(warp * 16 + g) * AD + 8 * i + 2 * qd + 1] = oacc[i][1];
      sm_o[(warp * 16 + g + 8) * AD + 8 * i + 2 * qd] = oacc[i][2];
      sm_o[(warp * 16 + g + 8) * AD + 8 * i + 2 * qd + 1] = oacc[i][3];
    }
    if (qd == 0) {
      sm_m[warp * 16 + g] = m0;
      sm_m[warp * 16 + g + 8] = m1;
      sm_l[warp * 16 + g] = l0;
      sm_l[warp * 16 + g + 8] = l1;
    }
    bar_consumers();
    for (int e = tid; e < hpc * AD; e += 128) {
      const int r = e / AD, d = e - r * AD;
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) mm = fmaxf(mm, sm_m[w * 16 + r]);
      float acc = 0.f, ll = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm_m[w * 16 + r];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - mm);
        acc += sm_o[(w * 16 + r) * AD + d] * f;
        ll += sm_l[w * 16 + r] * f;
      }
      if (nc == 1) {
        p.o[((size_t)b * p.H + h0 + r) * AD + d] = __float2bfloat16_rn(acc / ll);
        continue;
      }
      const size_t slot = ((size_t)b * p.H + h0 + r) * p.max_chunks + chunk;
      __stcg(part_o + slot * AD + d, acc);
      if (d == 0) {
        __stcg(part_ml + slot * 2, mm);
        __stcg(part_ml + slot * 2 + 1, ll);
      }
    }
    if (nc > 1) {
      bar_consumers();
      if (tid == 0) *s_last = (atom_add_acq_rel_gpu_s32(&p.counters[z], 1) == nc - 1);
      bar_consumers();
      if (*s_last) {
        for (int e = tid; e < hpc * AD; e += 128) {
          const int r = e / AD, d = e - r * AD;
          const size_t row = ((size_t)b * p.H + h0 + r) * p.max_chunks;
          float mm = -INFINITY;
          for (int c = 0; c < nc; ++c) mm = fmaxf(mm, __ldcg(part_ml + (row + c) * 2));
          float acc = 0.f, ll = 0.f;
          for (int c = 0; c < nc; ++c) {
            const float f = exp2f(__ldcg(part_ml + (row + c) * 2) - mm);
            ll += __ldcg(part_ml + (row + c) * 2 + 1) * f;
            acc += __ldcg(part_o + (row + c) * AD + d) * f;
          }
          p.o[((size_t)b * p.H + h0 + r) * AD + d] = __float2bfloat16_rn(acc / ll);
        }
        if (tid == 0) p.counters[z] = 0;
      }
    }
    bar_consumers();  // shared memory is reused by the next unit
  }
}

// ------------------------------------------------------------------ kernel

template <int MB>
__global__ void __launch_bounds__(160, 1)
    decode_block_kernel(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_o,
                        const __grid_constant__ CUtensorMap map_13, const __grid_constant__ CUtensorMap map_2,
                        const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ DecodeBlockParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  uint8_t* area = ring + STAGES * W_BYTES;
  float* os = reinterpret_cast<float*>(area + DB_AREA_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(os + 8 * MB * OS);
  uint64_t* empty = full + STAGES;
  unsigned long long* gbar = reinterpret_cast<unsigned long long*>(p.gbar);
  __shared__ int s_abort;
  __shared__ int s_last;
  __shared__ int s_qkv_done_word;
  int* s_qkv_done = &s_qkv_done_word;
  __shared__ float s_r[32];
  volatile int* abort_flag = &s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grid = gridDim.x, cta = blockIdx.x;
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    s_abort = 0;
    s_qkv_done_word = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    // One stream of 16 KB ring stages in the consumers' order: this CTA's
    // wqkv tiles, the K and V tiles of its attention units, then its wo, w1|w3
    // and w2 tiles. Weights never wait for the activations. A cache tile
    // that ends before the step's position holds rows written by earlier calls
    // and is loaded at once (during the wqkv phase); the tile holding the
    // position waits until the consumers have passed the barrier after wqkv,
    // whose epilogue writes that row.
    if (lane == 0) {
      const CUtensorMap* maps[4] = {&map_qkv, &map_o, &map_13, &map_2};
#pragma unroll
      for (int i = 0; i < 4; ++i) prefetch_tensormap(maps[i]);
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      int j = 0;
      bool ok = true, waited = false;
      // a free ring stage, armed for `bytes`; the previous kernel is waited for
      // once the first ring of weights is in flight
      auto next_stage = [&](uint32_t bytes) -> int {
        if (!waited && j == STAGES) {
          pdl_wait();
          pdl_trigger();
          waited = true;
        }
        const int st = j % STAGES;
        if (!wait_or_abort(&empty[st], ((j / STAGES) & 1) ^ 1, p.err, abort_flag)) return -1;
        mbar_arrive_expect_tx(&full[st], bytes);
        return st;
      };
      auto produce_linear = [&](int li) {
        const DbLinear& L = p.lin[li];
        int x, end;
        db_range(L, cta, grid, x, end);
        if (x >= end) return;
        const DbStage S = db_locate(L, x);
        int rb = S.rb, kl = x - S.reg_beg, sl = S.s, start = S.start, len = S.len;
        for (; x < end; ++x, ++j) {
          const int st = next_stage(W_BYTES);
          if (st < 0) {
            ok = false;
            return;
          }
          // the library's weight tiles: tile (rb, k stage) at rows (rb * NK + k stage) * 128 of the map
          tma_load_2d(ring + st * W_BYTES, maps[li], &full[st], 0, (rb * L.NK + start + kl) * RPC);
          if (++kl == len) {
            kl = 0;
            if (++rb == L.RB) {
              rb = 0;
              ++sl;
              start = db_slice_start(L, sl);
              len = db_slice_start(L, sl + 1) - start;
            }
          }
        }
      };
      produce_linear(0);
      if (ok && !waited) {
        pdl_wait();
        pdl_trigger();
        waited = true;
      }
      const int units = p.M * p.Hkv * ((p.H / p.Hkv) / p.hpc) * p.max_chunks;
      bool fresh = false;  // the row at the position is visible to this thread's TMA reads
      for (int u = cta; ok && u < units; u += grid) {
        DbUnit w;
        if (!db_unit(p, u, w)) continue;
        for (int jt = 0; ok && jt < w.n_tiles; ++jt) {
          const int key0 = w.k_begin + jt * AKT;
          if (!fresh && key0 + AKT > w.sp) {
            const uint64_t t0 = global_timer_ns();
            while (!ld_acquire_cta_shared(s_qkv_done)) {
              if (*abort_flag || global_timer_ns() - t0 > LLAMA_WAIT_LIMIT_NS) {
                if (!*abort_flag) atomicOr(p.err, LLAMA_DEV_TIMEOUT);
                *abort_flag = 1;
                ok = false;
                break;
              }
            }
            if (!ok) break;
            fence_proxy_async_global();
            fresh = true;
          }
          for (int kv = 0; kv < 2; ++kv, ++j) {
            const int st = next_stage(W_BYTES);
            if (st < 0) {
              ok = false;
              break;
            }
            const CUtensorMap* m = kv ? &map_v : &map_k;
            tma_load_2d(ring + st * W_BYTES, m, &full[st], 0, (int)(w.row0 + jt * AKT));
            tma_load_2d(ring + st * W_BYTES + 8192, m, &full[st], 64, (int)(w.row0 + jt * AKT));
          }
        }
      }
      for (int li = 1; li < 4 && ok; ++li) produce_linear(li);
      if (!waited) {
        pdl_wait();
        pdl_trigger();
      }
      // the CTA must not retire while a copy into its shared memory is in flight
      for (int i = (j > STAGES ? j - STAGES : 0); i < j; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.err);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  pdl_wait();
  pdl_trigger();
  int j = 0;
  if (!p.norm_local) {
    db_sumsq_phase(p, cta, grid);
    db_grid_sync(gbar, grid, p.err, abort_flag);
  }
  db_linear_phase<MB>(p, 0, cta, grid, j, ring, area, os, full, empty, abort_flag, &s_last, s_r);
  db_grid_sync(gbar, grid, p.err, abort_flag);
  if (tid == 0) st_release_cta_shared(s_qkv_done, 1);
  db_attention_phase(p, cta, grid, j, ring, area, full, empty, abort_flag, &s_last);
  db_grid_sync(gbar, grid, p.err, abort_flag);
  db_linear_phase<MB>(p, 1, cta, grid, j, ring, area, os, full, empty, abort_flag, &s_last, s_r);
  db_grid_sync(gbar, grid, p.err, abort_flag);
  db_linear_phase<MB>(p, 2, cta, grid, j, ring, area, os, full, empty, abort_flag, &s_last, s_r);
  db_grid_sync(gbar, grid, p.err, abort_flag);
  db_linear_phase<MB>(p, 3, cta, grid, j, ring, area, os, full, empty, abort_flag, &s_last, s_r);
}

// Self-test of the grid barrier's bound: two CTAs of 128 threads, CTA 1 never
// arrives, so CTA 0's wait runs out after the limit, records the timeout and
// returns; elapsed[0] receives the time CTA 0 spent in the barrier.
__global__ void __launch_bounds__(128) grid_barrier_selftest_kernel(unsigned long long* gbar, int* err,
                                                                    unsigned long long* elapsed) {
  __shared__ int s_abort;
  if (threadIdx.x == 0) s_abort = 0;
  __syncthreads();
  if (blockIdx.x == 1) return;
  const uint64_t t0 = global_timer_ns();
  db_grid_sync(gbar, 2, err, &s_abort);
  if (threadIdx.x == 0) elapsed[0] = global_timer_ns() - t0;
}

cudaError_t launch_grid_barrier_selftest(void* gbar, int* err, unsigned long long* elapsed, cudaStream_t st) {
  grid_barrier_selftest_kernel<<<2, 128, 0, st>>>(reinterpret_cast<unsigned long long*>(gbar), err, elapsed);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ host side

static size_t db_smem(int mb) {
  return 1024 + (size_t)STAGES * W_BYTES + DB_AREA_BYTES + (size_t)8 * mb * OS * 4 + 2 * STAGES * 8 + 16;
}

static DbLinear db_plan_linear(int M, int N, int K, int grid) {
  DbLinear L;
  L.N = N;
  L.K = K;
  L.RB = N / RPC;
  L.NK = K / KB;
  L.total = L.RB * L.NK;
  L.S = 1;
  // the smallest number of k slices whose x slice fits the shared-memory area
  while (L.S < L.NK && (size_t)M * ((size_t)((L.NK + L.S - 1) / L.S) * KB + 8) * 2 > DB_AREA_BYTES) ++L.S;
  (void)grid;
  return L;
}

DecodeBlockPlan plan_decode_block(int M, int dim, int H, int Hkv, int D, int F, int S_max, int max_len,
                                  int num_sms) {
  DecodeBlockPlan pl;
  pl.ok = false;
  const int n_rep = H / Hkv;
  if (M < 1 || M > 32 || D != AD || dim % RPC || ((H + 2 * Hkv) * D) % RPC || F % KB || (H * D) % KB) return pl;
  const int hpc = n_rep < 16 ? n_rep : 16;
  if (n_rep % hpc) return pl;
  pl.grid = num_sms;
  const int Ns[4] = {(H + 2 * Hkv) * D, dim, 2 * F, dim};
  const int Ks[4] = {dim, H * D, dim, F};
  size_t part = 0;
  int counters = 0;
  for (int i = 0; i < 4; ++i) {
    DbLinear& L = pl.lin[i];
    L = db_plan_linear(M, Ns[i], Ks[i], pl.grid);
    if ((long long)L.total * (pl.grid + 1) >= (1LL << 31)) return pl;  // index math is 32-bit
    if ((size_t)M * ((size_t)((L.NK + L.S - 1) / L.S) * KB + 8) * 2 > DB_AREA_BYTES) return pl;
    int maxc = 1;
    for (int rb = 0; rb < L.RB; ++rb) {
      const int c = db_contributors(L, rb, pl.grid, 0, 0, nullptr);
      if (c > maxc) maxc = c;
    }
    const size_t need = (size_t)maxc * M * L.N;
    if (need > part) part = need;
    if (L.RB > counters) counters = L.RB;
  }
  // attention: about one work unit per CTA, chunks of at least 128 keys
  pl.hpc = hpc;
  const int Z = M * Hkv * (n_rep / hpc);
  int want = pl.grid / Z;  // chunks per (sequence, head group): at most one unit per CTA
  if (want < 1) want = 1;
  int ck = (max_len + want - 1) / want;
  ck = (ck + AKT - 1) / AKT * AKT;
  if (ck < 128) ck = 128;
  pl.CK = ck;
  pl.max_chunks = (max_len + ck - 1) / ck;
  const size_t att = (size_t)M * H * pl.max_chunks * (AD + 2);
  if (att > part) part = att;
  if (Z > counters) counters = Z;
  pl.part_floats = part;
  pl.norm_local = pl.lin[0].S == 1 && pl.lin[2].S == 1;
  pl.counters = counters;
  pl.ok = true;
  return pl;
}

// Host-side walk of a plan with the kernel's own index functions (the
// producer's cursor and the consumers' segments): every stage of every linear
// belongs to one CTA; the cursor's tile equals db_locate's at every stage;
// tiles lie inside the weight matrix; a CTA's x slice fits the shared area;
// each row block's partial slots are 0 .. count-1 and fit the workspace; the
// attention's partials and counters fit too.
bool check_decode_block_plan(const DecodeBlockPlan& pl, int M, int H, size_t part_floats, int counters_n) {
  if (!pl.ok) return false;
  const int grid = pl.grid;
  for (int li = 0; li < 4; ++li) {
    const DbLinear& L = pl.lin[li];
    std::vector<int> seen(L.total, 0);
    std::vector<std::vector<int>> slots(L.RB);
    std::vector<int> counts(L.RB, -1);
    for (int cta = 0; cta < grid; ++cta) {
      int x, end;
      db_range(L, cta, grid, x, end);
      if (x >= end) continue;
      DbStage S = db_locate(L, x);
      int rb = S.rb, kl = x - S.reg_beg, sl = S.s, start = S.start, len = S.len;  // the producer's cursor
      int seg_first = x;
      for (; x < end; ++x) {
        const DbStage T = db_locate(L, x);
        if (T.rb != rb || T.start + (x - T.reg_beg) != start + kl) return false;
        if (rb >= L.RB || start + kl >= L.NK) return false;
        if ((size_t)M * ((size_t)T.len * 64 + 8) * 2 > DB_AREA_BYTES) return false;
        ++seen[x];
        const bool seg_ends = x + 1 == end || x + 1 == T.reg_beg + T.len;
        if (seg_ends) {
          const bool whole = L.S == 1 && seg_first == T.reg_beg && x + 1 == T.reg_beg + T.len;
          if (!whole) {
            int slot = 0;
            const int count = db_contributors(L, T.rb, grid, T.s, cta, &slot);
            if (slot < 0 || slot >= count || (size_t)count * M * L.N > part_floats) return false;
            if (counts[T.rb] >= 0 && counts[T.rb] != count) return false;
            counts[T.rb] = count;
            slots[T.rb].push_back(slot);
          }
          seg_first = x + 1;
        }
        if (++kl == len) {
          kl = 0;
          if (++rb == L.RB) {
            rb = 0;
            ++sl;
            start = db_slice_start(L, sl);
            len = db_slice_start(L, sl + 1) - start;
          }
        }
      }
    }
    for (int v : seen)
      if (v != 1) return false;
    for (int r = 0; r < L.RB; ++r) {
      if (counts[r] < 0) continue;
      std::vector<int> v = slots[r];
      std::sort(v.begin(), v.end());
      if ((int)v.size() != counts[r]) return false;
      for (int i = 0; i < counts[r]; ++i)
        if (v[i] != i) return false;
    }
    if (L.RB > counters_n) return false;
  }
  if ((size_t)M * H * pl.max_chunks * (AD + 2) > part_floats) return false;
  return true;
}

// A cooperative launch: the grid barriers need every CTA resident at once, and
// the driver then guarantees it (or refuses the launch). The grid is checked
// against the kernel's occupancy first, so a grid that cannot be resident is
// refused before anything runs.
template <int MB>
static cudaError_t db_launch(const CUtensorMap* maps, const DecodeBlockParams& p, int grid, cudaStream_t st) {
  const size_t smem = db_smem(MB);
  static std::atomic<unsigned long long> attr{0};
  cudaError_t e = ensure_smem(decode_block_kernel<MB>, smem, attr);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_block_kernel<MB>, 160, smem)) != cudaSuccess)
    return e;
  if ((long long)per_sm * sms < grid) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(160);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeCooperative;
  la[0].val.cooperative = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_block_kernel<MB>, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
}

cudaError_t launch_decode_block(const CUtensorMap* maps, const DecodeBlockParams& p, int grid, cudaStream_t st) {
  switch ((p.M + 7) / 8) {
    case 1: return db_launch<1>(maps, p, grid, st);
    case 2: return db_launch<2>(maps, p, grid, st);
    case 3: return db_launch<3>(maps, p, grid, st);
    default: return db_launch<4>(maps, p, grid, st);
  }
}

size_t decode_block_smem(int M) { return db_smem((M + 7) / 8); }

}  // namespace llama
