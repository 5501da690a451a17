// Next-token selection on the device: greedy argmax, or the top-p sampling of
// the LLaMA model.py walk-through (linkmax.top), section 3.3 generate /
// sample_top_p: probs = softmax(logits / temperature); sort descending; keep
// the tokens whose more-probable predecessors sum to at most top_p (mask
// cum - p > top_p); renormalise; draw one token from the kept set.
//
// The draw takes a caller-supplied uniform u in [0, 1) and returns the first
// token, in descending-probability order, at which the cumulative kept mass
// exceeds u times the kept total (inverse CDF). No sort is needed: the kept
// set is {i : p_i >= x*} for the smallest float x* whose strictly-larger mass
// is <= top_p, and the drawn token has the probability y* = the smallest float
// whose strictly-larger kept mass is <= t = u * kept total; both are found by
// bisection over the order of positive float bit patterns, each step one
// block-wide sum. Tokens with exactly equal probability are taken in index
// order.
#include "kernels.cuh"

namespace llama {

namespace {
constexpr int ST = 1024;  // threads per sequence
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll 1
  for (int w = 0; w < ST / 32; ++w) s += red[w];  // same order in every thread
  return s;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < ST / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// mass of the probabilities strictly above x (only those >= floor_x count)
__device__ __forceinline__ float mass_above(const float* p, int V, float x, float floor_x, float* red) {
  float s = 0.f;
  for (int i = threadIdx.x; i < V; i += ST) {
    const float v = p[i];
    if (v > x && v >= floor_x) s += v;
  }
  return block_sum(s, red);
}

// smallest positive float x with mass_above(x) <= target (bisection on bit patterns)
__device__ float bisect_threshold(const float* p, int V, float target, float floor_x, float* red) {
  uint32_t lo = 0u, hi = __float_as_uint(1.0f);  // mass_above(1.0) == 0 <= target
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (mass_above(p, V, __uint_as_float(mid), floor_x, red) <= target)
      hi = mid;
    else
      lo = mid + 1;
  }
  return __uint_as_float(lo);
}

// one CTA per sequence; logits [B][V] (row stride V); writes out[b * out_stride]
// unless keep[b * keep_stride] is set (then the token already there stays).
// With col (a captured decode step) out and keep move by *col columns and the
// uniforms by *col rows of B.
__global__ void __launch_bounds__(ST) sample_kernel(const float* __restrict__ logits, int V, float temperature,
                                                    float top_p, const float* __restrict__ uniforms,
                                                    float* __restrict__ scratch, int32_t* __restrict__ out,
                                                    int out_stride, const uint8_t* __restrict__ keep,
                                                    int keep_stride, const int* col) {
  pdl_wait();
  pdl_trigger();
  if (col) {
    const int c0 = *col;
    out += c0;
    if (keep) keep += c0;
    if (uniforms) uniforms += (size_t)c0 * gridDim.x;
  }
  __shared__ float red[ST / 32];
  __shared__ int red_i[ST / 32];
  const int b = blockIdx.x;
  const float* l = logits + (size_t)b * V;
  if (keep && keep[(size_t)b * keep_stride]) return;  // a prompt token: keep it (uniform over the CTA)
  int chosen = 0;
  if (!(temperature > 0.f)) {
    // greedy: the largest logit, lowest index on ties
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < V; i += ST) {
      const float v = l[i];
      if (v > best) {
        best = v;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) {
        best = ov;
        bi = oi;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      red[threadIdx.x >> 5] = best;
      red_i[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float bb = red[0];
      int ii = red_i[0];
      for (int w = 1; w < ST / 32; ++w)
        if (red[w] > bb || (red[w] == bb && red_i[w] < ii)) {
          bb = red[w];
          ii = red_i[w];
        }
      out[(size_t)b * out_stride] = ii;
    }
    return;
  }
  // probabilities softmax(l / temperature) into scratch
  float* p = scratch + (size_t)b * V;
  float m = -INFINITY;
  for (int i = threadIdx.x; i < V; i += ST) m = fmaxf(m, l[i]);
  m = block_max(m, red);
  const float inv_t = 1.f / temperature;
  float z = 0.f;
  for (int i = threadIdx.x; i < V; i += ST) {
    const float e = expf((l[i] - m) * inv_t);
    p[i] = e;
    z += e;
  }
  z = block_sum(z, red);
  const float inv_z = 1.f / z;
  for (int i = threadIdx.x; i < V; i += ST) p[i] *= inv_z;
  __syncthreads();
  // kept set: p_i >= x_keep
  const float x_keep = bisect_threshold(p, V, top_p, 0.f, red);
  const float kept = mass_above(p, V, -1.f, x_keep, red);
  const float t = uniforms[b] * kept;
  // the drawn probability value, then the tied token in index order
  const float y = bisect_threshold(p, V, t, x_keep, red);
  const float above = mass_above(p, V, y, x_keep, red);
  const int k = min((int)((t - above) / y), V);  // 0-based among tokens with p == y
  // the k-th index with p == y (scan in index order, chunk by chunk)
  __shared__ int s_count[ST / 32];
  __shared__ int s_found;
  if (threadIdx.x == 0) s_found = -1;
  int base_count = 0;
  for (int c0 = 0; c0 < V; c0 += ST) {
    const int i = c0 + threadIdx.x;
    const bool hit = i < V && p[i] == y;
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if ((threadIdx.x & 31) == 0) s_count[threadIdx.x >> 5] = __popc(bal);
    __syncthreads();
    int before = base_count, total = 0;
    for (int w = 0; w < ST / 32; ++w) {
      if (w < (threadIdx.x >> 5)) before += s_count[w];
      total += s_count[w];
    }
    before += __popc(bal & ((1u << (threadIdx.x & 31)) - 1u));
    if (hit && before == k) s_found = i;
    __syncthreads();
    if (s_found >= 0) break;
    base_count += total;
    __syncthreads();
  }
  chosen = s_found;
  if (chosen < 0) {
    // k ran past the last tied token (rounding at the very end of the range): take the last one
    int last = -1;
    for (int i = threadIdx.x; i < V; i += ST)
      if (p[i] == y) last = max(last, i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    if ((threadIdx.x & 31) == 0) red_i[threadIdx.x >> 5] = last;
    __syncthreads();
    for (int w = 0; w < ST / 32; ++w) chosen = max(chosen, red_i[w]);
  }
  if (threadIdx.x == 0) out[(size_t)b * out_stride] = chosen;
}

cudaError_t launch_sample(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                          float* scratch, int32_t* out, int out_stride, const uint8_t* keep, int keep_stride,
                          cudaStream_t st, const int* col) {
  return launch_pdl(sample_kernel, dim3(B), dim3(ST), 0, st, logits, V, temperature, top_p, uniforms, scratch, out,
                    out_stride, keep, keep_stride, col);
}

}  // namespace llama
