// Device-side helpers shared by the kernels of the LLaMA decoder-block library:
// numeric conversions, the epilogue parameter block, and thin inline-PTX
// wrappers for mbarriers, TMA bulk copies and the tcgen05 tensor-core ops of
// sm_100a. Every wait on an mbarrier is bounded: after LLAMA_WAIT_LIMIT_NS of
// global-timer time it records LLAMA_DEV_TIMEOUT in the error word and the
// caller unwinds instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "llama_b200.h"

#define LLAMA_DEV_TOKEN_RANGE 1
#define LLAMA_DEV_POS_RANGE 2
#define LLAMA_DEV_TIMEOUT 4

// about one second of waiting before an mbarrier wait gives up
#ifndef LLAMA_WAIT_LIMIT_NS
#define LLAMA_WAIT_LIMIT_NS 1000000000ull
#endif

typedef __nv_bfloat16 bf16;

namespace llama {

// ---------------------------------------------------------------- conversions

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// round through the storage type (identity for fp32)
template <typename T> __device__ __forceinline__ float round_to(float x) { return to_f32(from_f32<T>(x)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// (a, b) = hi + lo with hi = bf16(a, b) and lo = bf16 of the remainders
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  const float2 h = unpack_bf16x2(hi);
  lo = pack_bf16x2(a - h.x, b - h.y);
}

// store 8 consecutive values (fp32 in registers) to storage type T
__device__ __forceinline__ void store8(float* dst, const float* v) {
  float4* d = reinterpret_cast<float4*>(dst);
  d[0] = make_float4(v[0], v[1], v[2], v[3]);
  d[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(bf16* dst, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}
__device__ __forceinline__ void store4(float* dst, const float* v) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16* dst, const float* v) {
  uint2 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  *reinterpret_cast<uint2*>(dst) = u;
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + __expf(-a)); }

// ---------------------------------------------------------------- epilogues
//
// Every GEMM path (tcgen05, decode GEMV, fp32 SIMT) hands its fp32 results to
// the same epilogue in chunks of 8 consecutive output columns of one row.

enum EpiKind : int {
  EPI_QKV_ROPE = 0,   // RoPE on q and k pairs, q -> q_out, k/v -> cache slot
  EPI_RESIDUAL = 1,   // h[m, n] += acc  (fp32 residual stream)
  EPI_SWIGLU = 2,     // packed w1/w3 rows (2j, 2j+1): g[m, j] = silu(a) * b
  EPI_STORE_F32 = 3,  // out[m, n] = acc (logits, plain linear)
};

struct EpiParams {
  int kind;
  int M, N;
  // EPI_QKV_ROPE
  void* q_out;             // [M, H*D] activation dtype
  void* cache_k;           // this layer's cache [B_max][Hkv][S_max][D]
  void* cache_v;
  const float2* rope;      // [2*S_max][D/2] (cos, sin)
  const int* start_pos;    // [B] device positions, or nullptr -> start_pos_scalar
  int start_pos_scalar;
  int T;                   // tokens per sequence: row m -> (b = m / T, s = m % T)
  int H, Hkv, D, S_max;
  // EPI_RESIDUAL / EPI_STORE_F32
  float* out;              // [M, ld_out]
  long long ld_out;
  // EPI_SWIGLU
  void* g_out;             // [M, N/2] activation dtype
  int* err;
};

template <typename T>
__device__ __forceinline__ void epilogue8(const EpiParams& p, int m, int n0, float* v) {
  switch (p.kind) {
    case EPI_QKV_ROPE: {
      const int D = p.D, HD = p.H * D, KD = p.Hkv * D;
      const int b = m / p.T, s = m - b * p.T;
      const int pos = (p.start_pos ? p.start_pos[b] : p.start_pos_scalar) + s;
      if (pos < 0 || pos >= p.S_max) {
        atomicOr(p.err, LLAMA_DEV_POS_RANGE);
        return;
      }
      const int d0 = n0 % D;
      if (n0 < HD + KD) {
        const float2* cs = p.rope + (size_t)pos * (D / 2) + d0 / 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 c = cs[i];
          const float x = v[2 * i], y = v[2 * i + 1];
          v[2 * i] = x * c.x - y * c.y;
          v[2 * i + 1] = y * c.x + x * c.y;
        }
      }
      if (n0 < HD) {
        store8(reinterpret_cast<T*>(p.q_out) + (size_t)m * HD + n0, v);
      } else {
        const bool is_k = n0 < HD + KD;
        const int kvh = (n0 - HD - (is_k ? 0 : KD)) / D;
        T* cache = reinterpret_cast<T*>(is_k ? p.cache_k : p.cache_v);
        const size_t slot = (((size_t)b * p.Hkv + kvh) * p.S_max + pos) * D + d0;
        store8(cache + slot, v);
      }
      break;
    }
    case EPI_RESIDUAL: {
      float* dst = p.out + (size_t)m * p.ld_out + n0;
      float4* d4 = reinterpret_cast<float4*>(dst);
      float4 a = d4[0], c = d4[1];
      a.x += v[0]; a.y += v[1]; a.z += v[2]; a.w += v[3];
      c.x += v[4]; c.y += v[5]; c.z += v[6]; c.w += v[7];
      d4[0] = a;
      d4[1] = c;
      break;
    }
    case EPI_SWIGLU: {
      float g[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) g[i] = silu_f(v[2 * i]) * v[2 * i + 1];
      store4(reinterpret_cast<T*>(p.g_out) + (size_t)m * (p.N / 2) + n0 / 2, g);
      break;
    }
    default: {
      store8(p.out + (size_t)m * p.ld_out + n0, v);
      break;
    }
  }
}

// ---------------------------------------------------------------- PTX wrappers

// Programmatic dependent launch: every kernel of the forward pass is launched
// so that it may start while the previous one drains. pdl_wait blocks until
// the previous kernel has completed and its writes are visible; pdl_trigger
// (always called after pdl_wait) then lets the next kernel begin launching.
// Hence when a kernel starts, every kernel before its immediate predecessor
// has completed. Before pdl_wait a kernel may only read weights, tensor maps,
// positions (inputs of the call, or written by the embedding kernel of a
// captured generation step, which is at least three launches before any kernel
// that reads them early) and, for the decode attention, cache slots written by
// calls before the predecessor; it never writes global memory there.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait until the phase with the given parity has completed. Returns false
// (and records a timeout) if that takes longer than the wait limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > LLAMA_WAIT_LIMIT_NS) {
      atomicOr(err, LLAMA_DEV_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait that also gives up as soon as another role of the CTA has given
// up (abort_flag in shared memory), so one timeout unwinds the whole CTA quickly.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > LLAMA_WAIT_LIMIT_NS) {
      atomicOr(err, LLAMA_DEV_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Arrival on a global counter with acquire-release semantics at GPU scope:
// releases this thread's earlier writes and the writes of its CTA ordered
// before it by a bar.sync, and acquires the writes released by the arrivals
// before it (one L2 round trip where a fence plus an atomic takes two).
__device__ __forceinline__ int atomic_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Flag store with release semantics and load with acquire semantics, GPU scope.
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory, completing
// on an mbarrier with a transaction-byte count.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Plain bulk copy of `bytes` contiguous bytes global -> this CTA's shared memory,
// completing on `bar` (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 (5th-generation tensor cores, accumulators in tensor memory)

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate, one CTA.
__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Each thread of a warp reads 32 consecutive fp32 columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 64 bf16 (128 B), 8-row atoms of 1024 B.
// Fields: start address >> 4 [0,14), leading-dim byte offset >> 4 [16,30)
// (unused for swizzled K-major, set to 1), stride-dim byte offset >> 4
// [32,46) = 1024 >> 4, descriptor version 1 [46,48), swizzle mode 2 =
// 128-byte [61,64).
__device__ __forceinline__ uint64_t make_sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at
// bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---- legacy warp-level MMA (used for the HBM-bound decode GEMV and attention)

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// 16-byte global load that does not allocate in L1 (streamed weights)
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// CTA pairs (clusters of two on an SM pair) and the 2-SM tcgen05 forms: one
// thread of the rank-0 CTA issues MMAs with M = 256 over both CTAs, each CTA
// supplying its half of A (its 128 rows) and of B (half the N columns) from its
// own shared memory or TMEM; copies into either CTA can complete on rank 0's
// barriers; commits arrive on the barriers of both CTAs.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// every thread of both CTAs (release / acquire at cluster scope)
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// arrive on the barrier at the same shared-memory offset in CTA `rank` of the
// cluster, relaxed (no release fence): for arrivals that announce work already
// complete when they are made (tensor-memory stores or loads the arriving
// threads have waited for with tcgen05.wait::st / ::ld), so only the signal has
// to travel.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}
// wait for a phase of a local barrier that the other CTA of the pair arrives on
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool wait_cluster_or_abort(uint64_t* bar, uint32_t parity, int* err,
                                                      volatile int* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  if (*abort_flag) return false;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > LLAMA_WAIT_LIMIT_NS) {
      atomicOr(err, LLAMA_DEV_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
// shared::cluster address of the barrier at the same offset in CTA `rank`
__device__ __forceinline__ uint32_t mbar_cluster_addr(uint64_t* bar, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(bar)), "r"(rank));
  return ra;
}
// 2-D TMA load into this CTA's shared memory whose bytes complete on a barrier
// that may sit in either CTA of the pair (the 2-SM form; no multicast)
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
// the 3-D form of the same
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 2-SM MMA (M = 256 over the pair), A by descriptor / A from TMEM, B by descriptor
__device__ __forceinline__ void mma2_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma2_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive on `bar` in both CTAs of the pair once every MMA issued so far has finished
__device__ __forceinline__ void commit2(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"((unsigned short)3)
               : "memory");
}
// instruction descriptor, kind::f16, bf16 A and B, fp32 D, M rows over the pair
__host__ __device__ constexpr uint32_t idesc2_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}


}  // namespace llama
