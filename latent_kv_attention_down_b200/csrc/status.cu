// The library's device status word and the self-test of the bounded waits.
#include <mutex>

#include "kernels.h"
#include "ptx.cuh"

namespace vmla {

__device__ unsigned g_device_error;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned* g_err_word[kMaxDevices] = {};
}  // namespace

// Looked up with cudaGetSymbolAddress the first time per device, with that device current, and
// kept: later calls (a stream capture among them) make no CUDA call here but cudaGetDevice.
unsigned* device_error_word() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_word[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_word[dev] = static_cast<unsigned*>(p);
  }
  return g_err_word[dev];
}

namespace {
// One thread waits on an mbarrier that nothing arrives at; the bounded wait must
// give up after limit_ns, record DEV_ERR_TIMEOUT_SELFTEST and return.
__global__ void selftest_wait_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Guard g{&abort_flag, err, limit_ns};
    wait_phase(&bar, 0, g, DEV_ERR_TIMEOUT_SELFTEST);
  }
  __syncthreads();
}
}  // namespace

namespace {
__global__ void selftest_exp2_kernel(const float2* x, float2* y, int64_t pairs) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < pairs) y[i] = exp2_poly2(x[i]);
}
}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y, int64_t n, cudaStream_t s) {
  const int64_t pairs = n / 2;
  if (pairs == 0) return cudaSuccess;
  selftest_exp2_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(reinterpret_cast<const float2*>(x),
                                                                        reinterpret_cast<float2*>(y), pairs);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(unsigned* err, uint64_t limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace vmla
