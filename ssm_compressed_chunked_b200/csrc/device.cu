// Per-device launch facts the launchers need, computed once per device and
// safe to query from several host threads: the SM count, and whether a
// kernel's dynamic shared-memory limit has been raised on the device.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kMaxDevices = 64;
constexpr int kMaxKernels = 8;
std::mutex g_mu;
int g_sms[kMaxDevices] = {};
const void* g_raised[kMaxDevices][kMaxKernels] = {};
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[dev] == 0) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = sms > 0 ? sms : 148;
  }
  return g_sms[dev];
}

cudaError_t raise_smem_limit(const void* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int k = 0; k < kMaxKernels; ++k) {
    if (g_raised[dev][k] == kernel) return cudaSuccess;
    if (g_raised[dev][k] == nullptr) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) g_raised[dev][k] = kernel;
      return e;
    }
  }
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

namespace {
// The give-up path every pipeline wait has, exercised on purpose: nothing ever arrives on `bar`, so
// the bounded wait runs out after limit_ns and the status bit is raised; the kernel then returns.
__global__ void wait_selftest_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns)) raise_status(status, ATTAMBA_DEV_TIMEOUT);
}
}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace attamba
