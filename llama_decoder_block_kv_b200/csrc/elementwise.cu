// Memory-bound kernels around the GEMMs: the token-embedding gather, RMSNorm,
// weight packing at load time and the cache layout converters.
#include "kernels.cuh"

namespace llama {

// ---------------------------------------------------------------------------
// Token embedding ("LLaMA: Open and Efficient Foundation Language Models"
// notes, Transformer.forward: h = tok_embeddings(tokens)). One CTA per token;
// the table row (act type) is widened to the fp32 residual stream. An id
// outside [0, vocab) raises the token-range flag and yields a zero row.
// With col (a captured decode step, T_ = 1) the token of sequence b is
// tokens[b * tok_stride + *col] and CTA b also records its position, *col, in
// pos[b] for the blocks that follow.
template <typename T>
__global__ void embed_gather_kernel(const int* __restrict__ tokens, const T* __restrict__ table,
                                    float* __restrict__ h, int dim, int vocab, int T_, int tok_stride, int* err,
                                    const int* col, int* pos) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;  // token b * T_ + s, read from tokens[b * tok_stride + s]
  const int c0 = col ? *col : 0;
  if (col && pos && threadIdx.x == 0) pos[t] = c0;
  const int id = tokens[(t / T_) * tok_stride + t % T_ + c0];
  float* dst = h + (size_t)t * dim;
  if (id < 0 || id >= vocab) {
    if (threadIdx.x == 0) atomicOr(err, LLAMA_DEV_TOKEN_RANGE);
    for (int i = threadIdx.x * 4; i < dim; i += blockDim.x * 4)
      *reinterpret_cast<float4*>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const T* src = table + (size_t)id * dim;
  for (int i = threadIdx.x * 8; i < dim; i += blockDim.x * 8) {
    float v[8];
    if constexpr (sizeof(T) == 2) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + i);
      float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z), d = unpack_bf16x2(u.w);
      v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
    } else {
      const float4 a = *reinterpret_cast<const float4*>(src + i);
      const float4 b = *reinterpret_cast<const float4*>(src + i + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    store8(dst + i, v);
  }
}

// ---------------------------------------------------------------------------
// RMSNorm, the notes' RMSNorm.forward: _norm(x.float()).type_as(x) * weight,
// _norm(x) = x * rsqrt(mean(x^2) + eps). The statistics are fp32; the
// normalised row is rounded to the act type, multiplied by the weight and
// rounded again. One CTA per row, 16-byte loads, warp-shuffle then
// shared-memory reduction. ``rows`` optionally maps output row r to input row
// rows[r] (the LM head of the last position only).
template <typename T, int THREADS>
__global__ void __launch_bounds__(THREADS) rmsnorm_kernel(const float* __restrict__ h, const T* __restrict__ w,
                                                          T* __restrict__ out, int dim, float eps, int in_row_stride_T,
                                                          int in_row_offset) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const float* x = h + ((size_t)r * in_row_stride_T + in_row_offset) * dim;
  __shared__ float red[THREADS / 32];
  float ss = 0.f;
  for (int i = threadIdx.x * 4; i < dim; i += THREADS * 4) {
    const float4 a = *reinterpret_cast<const float4*>(x + i);
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float s = threadIdx.x < THREADS / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) red[0] = s;
  }
  __syncthreads();
  const float inv = rsqrtf(red[0] / (float)dim + eps);
  T* y = out + (size_t)r * dim;
  for (int i = threadIdx.x * 4; i < dim; i += THREADS * 4) {
    const float4 a = *reinterpret_cast<const float4*>(x + i);
    float v[4] = {a.x, a.y, a.z, a.w};
    float wv[4];
    if constexpr (sizeof(T) == 2) {
      const uint2 u = *reinterpret_cast<const uint2*>(w + i);
      const float2 p = unpack_bf16x2(u.x), q = unpack_bf16x2(u.y);
      wv[0] = p.x; wv[1] = p.y; wv[2] = q.x; wv[3] = q.y;
    } else {
      const float4 q = *reinterpret_cast<const float4*>(w + i);
      wv[0] = q.x; wv[1] = q.y; wv[2] = q.z; wv[3] = q.w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = round_to<T>(v[j] * inv) * wv[j];
    store4(y + i, v);
  }
}

// ---------------------------------------------------------------------------
// Load-time packing of w1 and w3 [F][dim] into one [2F][dim] matrix whose row
// 2j is w1 row j and row 2j+1 is w3 row j, so that a GEMM output chunk holds
// matching gate/up columns side by side.
template <typename T>
__global__ void pack_w13_kernel(const T* __restrict__ w1, const T* __restrict__ w3, T* __restrict__ out, int F,
                                int dim) {
  const size_t row = blockIdx.x;  // 0 .. 2F-1
  const T* src = (row & 1) ? w3 + (row >> 1) * dim : w1 + (row >> 1) * dim;
  T* dst = out + row * dim;
  for (int i = threadIdx.x; i < dim; i += blockDim.x) dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// Weight tiles: the bf16 weights of a block are stored as contiguous 16 KB
// tiles of 128 rows x 64 k, tile (rb, kb) at index rb * (K/64) + kb, so each
// 128 x 64 operand stage of the GEMV and the tensor-core GEMM is one
// contiguous 16 KB read instead of 128 row pieces of 128 bytes. Element
// (n, k) goes to tile (n / 128, k / 64), row n % 128, column k % 64; rows past
// N are zero.
__global__ void tile_weights_kernel(const bf16* __restrict__ src, bf16* __restrict__ dst, int N, int K) {
  const int nk = K / 64;
  const size_t chunks = tiled_weight_elems(N, K) / 8;  // 16-byte pieces of the destination
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < chunks; c += (size_t)gridDim.x * blockDim.x) {
    const size_t e = c * 8;
    const size_t tile = e / (128 * 64);
    const int in_tile = (int)(e - tile * (128 * 64));
    const int r = in_tile / 64, col = in_tile % 64;
    const int rb = (int)(tile / nk), kb = (int)(tile - (size_t)rb * nk);
    const int n = rb * 128 + r, k = kb * 64 + col;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < N) v = *reinterpret_cast<const uint4*>(src + (size_t)n * K + k);
    *reinterpret_cast<uint4*>(dst + e) = v;
  }
}

void launch_tile_weights(const void* src, void* dst, int N, int K, cudaStream_t st) {
  tile_weights_kernel<<<1184, 256, 0, st>>>(reinterpret_cast<const bf16*>(src), reinterpret_cast<bf16*>(dst), N, K);
}

// ---------------------------------------------------------------------------
// Half-split RoPE weights (pairs (i, i + D/2) of each head) into the
// interleaved order the kernels rotate (pairs (2i, 2i+1)): row 2i of a head
// takes row i, row 2i+1 takes row i + D/2. q.k products are unchanged.
template <typename T>
__global__ void rope_rows_to_interleaved_kernel(const T* __restrict__ src, T* __restrict__ dst, int D, int dim) {
  const size_t r = blockIdx.x;  // destination row
  const int h = r / D, j = r % D;
  const T* s = src + ((size_t)h * D + (j & 1 ? D / 2 : 0) + (j >> 1)) * dim;
  T* d = dst + r * dim;
  for (int i = threadIdx.x; i < dim; i += blockDim.x) d[i] = s[i];
}

// position of element j of a head in the interleaved order, given its index j
// in the half-split order
__device__ __forceinline__ int half_split_to_interleaved(int j, int D) {
  return j < D / 2 ? 2 * j : 2 * (j - D / 2) + 1;
}

// ---------------------------------------------------------------------------
// Cache layout conversion between the library's [b][kvh][pos][D] and the
// pages' logical [b][pos][kvh][D] (the notes' Attention cache_k shape).
// half_split: the logical side holds the head dimension in half-split order.
template <typename T>
__global__ void kv_to_logical_kernel(const T* __restrict__ src, T* __restrict__ dst, int Bm, int S, int Hkv, int D,
                                     int to_logical, int half_split) {
  const size_t row = blockIdx.x;  // over Bm * S * Hkv rows of D
  const int kvh = row % Hkv;
  const size_t bp = row / Hkv;
  const int pos = bp % S;
  const int b = bp / S;
  const size_t lib = (((size_t)b * Hkv + kvh) * S + pos) * D;
  const size_t logi = row * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const int li = half_split ? half_split_to_interleaved(i, D) : i;  // library index of logical element i
    if (to_logical)
      dst[logi + i] = src[lib + li];
    else
      dst[lib + li] = src[logi + i];
  }
}

// ---------------------------------------------------------------------------
// host launchers

template <typename T>
cudaError_t launch_embed(const int* tokens, const void* table, float* h, int n_tok, int dim, int vocab, int T_,
                         int tok_stride, int* err, cudaStream_t st, const int* col, int* pos) {
  return launch_pdl(embed_gather_kernel<T>, dim3(n_tok), dim3(128), 0, st, tokens, reinterpret_cast<const T*>(table), h, dim,
             vocab, T_, tok_stride, err, col, pos);
}

// ---------------------------------------------------------------------------
// Step counter of a captured decode step: *col = value, or *col += 1 after the
// step's last kernel (one thread; ordered by the launch dependencies).
__global__ void step_counter_kernel(int* col, int value, int add) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) *col = add ? *col + 1 : value;
}

cudaError_t launch_step_counter(int* col, int value, int add, cudaStream_t st) {
  return launch_pdl(step_counter_kernel, dim3(1), dim3(32), 0, st, col, value, add);
}

template <typename T>
cudaError_t launch_rmsnorm(const float* h, const void* w, void* out, int rows, int dim, float eps,
                           int in_row_stride_T, int in_row_offset, cudaStream_t st) {
  if (dim >= 4096)  // one float4 per thread and pass at dim 4096 (a row is read in one round trip)
    return launch_pdl(rmsnorm_kernel<T, 1024>, dim3(rows), dim3(1024), 0, st, h, reinterpret_cast<const T*>(w),
               reinterpret_cast<T*>(out), dim, eps, in_row_stride_T, in_row_offset);
  else
    return launch_pdl(rmsnorm_kernel<T, 64>, dim3(rows), dim3(64), 0, st, h, reinterpret_cast<const T*>(w),
               reinterpret_cast<T*>(out), dim, eps, in_row_stride_T, in_row_offset);
}

template <typename T>
void launch_pack_w13(const void* w1, const void* w3, void* out, int F, int dim, cudaStream_t st) {
  pack_w13_kernel<T><<<2 * F, 256, 0, st>>>(reinterpret_cast<const T*>(w1), reinterpret_cast<const T*>(w3),
                                            reinterpret_cast<T*>(out), F, dim);
}

template <typename T>
void launch_kv_convert(const void* src, void* dst, int Bm, int S, int Hkv, int D, int to_logical, int half_split,
                       cudaStream_t st) {
  const size_t rows = (size_t)Bm * S * Hkv;
  kv_to_logical_kernel<T><<<(unsigned)rows, 128, 0, st>>>(reinterpret_cast<const T*>(src), reinterpret_cast<T*>(dst),
                                                          Bm, S, Hkv, D, to_logical, half_split);
}

template <typename T>
void launch_rope_rows_to_interleaved(const void* src, void* dst, int heads, int D, int dim, cudaStream_t st) {
  rope_rows_to_interleaved_kernel<T><<<heads * D, 256, 0, st>>>(reinterpret_cast<const T*>(src),
                                                                reinterpret_cast<T*>(dst), D, dim);
}

#define INST(T)                                                                                              \
  template cudaError_t launch_embed<T>(const int*, const void*, float*, int, int, int, int, int, int*,       \
                                       cudaStream_t, const int*, int*);                                  \
  template cudaError_t launch_rmsnorm<T>(const float*, const void*, void*, int, int, float, int, int,       \
                                         cudaStream_t);                                                   \
  template void launch_pack_w13<T>(const void*, const void*, void*, int, int, cudaStream_t);                 \
  template void launch_kv_convert<T>(const void*, void*, int, int, int, int, int, int, cudaStream_t);   \
  template void launch_rope_rows_to_interleaved<T>(const void*, void*, int, int, int, cudaStream_t);
INST(float)
INST(bf16)
#undef INST

}  // namespace llama
