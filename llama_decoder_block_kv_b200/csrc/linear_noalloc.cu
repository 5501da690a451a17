// llama_linear_noalloc: the decode GEMV of llama_linear (LLAMA_PATH_GEMV)
// with its scratch memory taken from a fixed array inside the library image
// instead of a cudaMalloc'd workspace.
//
// Who needs it: callers that must not allocate device memory at call time,
// e.g. a host application whose device memory is entirely carved up by its own
// pool allocator (a cudaMalloc behind its back can fail or fragment it), or a
// latency-critical loop where cudaMalloc/cudaFree are not acceptable because
// they can synchronise the device. The caller still passes x, w and y.
//
// The scratch (fp32 split-K partial sums, per-row-block arrival counters and an
// error word) lives in one file-scope __device__ array. Every GPU on which the
// library's device code is loaded holds it until the process exits. In host
// code the array's name only stands in for the symbol, so the device address is
// fetched with cudaGetSymbolAddress once per device, on the first call made
// while that device is current; that first call should therefore come before
// any stream capture. All calls on a device share the one array: calls whose
// kernels overlap on the GPU (e.g. on two streams) race and corrupt each
// other's partial sums. The counters are cleared on the caller's stream before
// each launch.
#include <cstring>
#include <mutex>

#include "kernels.cuh"

namespace llama {
namespace {

constexpr size_t NOALLOC_PART_FLOATS = (size_t)2 << 20;  // 2 Mi fp32 partial sums (8 MiB)
constexpr int NOALLOC_COUNTERS = 4096;                    // row blocks of 128 -> N <= 524288
constexpr size_t NOALLOC_BYTES = NOALLOC_PART_FLOATS * 4 + NOALLOC_COUNTERS * 4 + 256;
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char noalloc_scratch[NOALLOC_BYTES];

struct DeviceScratch {
  bool ready = false;
  unsigned char* ptr = nullptr;
};
DeviceScratch g_scratch[MAX_DEVICES];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up once per device).
int scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLAMA_ERR_CUDA;
  if (dev < 0 || dev >= MAX_DEVICES) return LLAMA_ERR_INVALID_ARGS;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch[dev].ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || p == nullptr) return LLAMA_ERR_CUDA;
    g_scratch[dev].ptr = static_cast<unsigned char*>(p);
    g_scratch[dev].ready = true;
  }
  *out = g_scratch[dev].ptr;
  return LLAMA_OK;
}

}  // namespace
}  // namespace llama

extern "C" int llama_linear_noalloc(const void* x, const void* w, float* y, int M, int N, int K, void* cuda_stream) {
  using namespace llama;
  if (!x || !w || !y || M < 1 || M > 32 || N < 8 || N % 8 || K < 64 || K % 64) return LLAMA_ERR_INVALID_ARGS;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLAMA_ERR_CUDA;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const GemvPlan p = plan_gemv(M, N, K, sms);
  if (p.part_floats > NOALLOC_PART_FLOATS || p.row_blocks > NOALLOC_COUNTERS) return LLAMA_ERR_TOO_LARGE;
  unsigned char* base = nullptr;
  int r = scratch_on_current_device(&base);
  if (r != LLAMA_OK) return r;
  float* part = reinterpret_cast<float*>(base);
  int* counters = reinterpret_cast<int*>(base + NOALLOC_PART_FLOATS * 4);
  int* err = counters + NOALLOC_COUNTERS;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
  // the arrival counters and the error word must start at zero
  if (cudaMemsetAsync(counters, 0, (NOALLOC_COUNTERS + 1) * sizeof(int), st) != cudaSuccess) return LLAMA_ERR_CUDA;
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.kind = EPI_STORE_F32;
  e.M = M;
  e.N = N;
  e.out = y;
  e.ld_out = N;
  e.err = err;
  if (launch_gemv_bf16(x, w, 0, M, N, K, p, part, counters, e, sms, st) != cudaSuccess) return LLAMA_ERR_CUDA;
  return LLAMA_OK;
}
