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
// each launch. The error word is not: a bounded wait that gave up leaves its bit
// there until llama_linear_noalloc_status reads and clears it. cudaDeviceReset
// unloads the array with the rest of the device code, so the address found at
// set-up is no longer valid on that device afterwards; a failed CUDA call in
// this path forgets the address, so the next call looks it up again.
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

// After a failed CUDA call the cached address may be stale (e.g. the device was
// reset): look it up again on the next call.
void forget_scratch_of_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  g_scratch[dev].ready = false;
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
  // the arrival counters must start at zero; the error word (bit 4: a bounded
  // wait timed out) is left as it is until llama_linear_noalloc_status clears it
  if (cudaMemsetAsync(counters, 0, NOALLOC_COUNTERS * sizeof(int), st) != cudaSuccess) {
    forget_scratch_of_current_device();
    return LLAMA_ERR_CUDA;
  }
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.kind = EPI_STORE_F32;
  e.M = M;
  e.N = N;
  e.out = y;
  e.ld_out = N;
  e.err = err;
  if (launch_gemv_bf16(x, w, 0, M, N, K, p, part, counters, e, sms, st) != cudaSuccess) {
    forget_scratch_of_current_device();
    return LLAMA_ERR_CUDA;
  }
  return LLAMA_OK;
}

extern "C" int llama_linear_noalloc_status(int* flags) {
  using namespace llama;
  if (flags) *flags = 0;
  unsigned char* base = nullptr;
  int r = scratch_on_current_device(&base);
  if (r != LLAMA_OK) return r;
  int* err = reinterpret_cast<int*>(base + NOALLOC_PART_FLOATS * 4) + NOALLOC_COUNTERS;
  int word = 0;
  // a plain synchronous copy into a host variable: nothing is allocated
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpy(&word, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(err, 0, sizeof(int)) != cudaSuccess) {
    forget_scratch_of_current_device();
    return LLAMA_ERR_CUDA;
  }
  if (flags) *flags = word;
  return (word & LLAMA_DEV_TIMEOUT) ? LLAMA_ERR_TIMEOUT : LLAMA_OK;
}
