// Per-device runtime state, status strings, the device error word and the
// failure-path test kernel.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "common.h"
#include "ptx.cuh"

namespace nvfp4 {

// One error word per device that loads the library.  Kernels receive its
// address as a parameter (the host never hands them the symbol itself).
__device__ unsigned g_device_error_word;

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];
std::atomic<uint64_t> g_timeout_ns{0};
std::atomic<int> g_decode_coop{0};
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s
constexpr uint64_t kMinDrainNs = 1000000000ull;        // 1 s

void init_device(int dev) {
  DeviceInfo& d = g_info[dev];
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_device_error_word) != cudaSuccess) return;
  d.sm_count = prop.multiProcessorCount;
  d.major = prop.major;
  d.minor = prop.minor;
  d.max_smem_optin = prop.sharedMemPerBlockOptin;
  d.err_word = static_cast<unsigned*>(addr);
  d.device = dev;
}
}  // namespace

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::call_once(g_once[dev], init_device, dev);
  if (g_info[dev].device != dev) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return &g_info[dev];
}

bool decode_cooperative() { return g_decode_coop.load(std::memory_order_relaxed) != 0; }

uint64_t wait_timeout_ns() {
  const uint64_t t = g_timeout_ns.load(std::memory_order_relaxed);
  return t ? t : kDefaultTimeoutNs;
}

uint64_t drain_timeout_ns() {
  const uint64_t t = wait_timeout_ns();
  return t > kMinDrainNs ? t : kMinDrainNs;
}

// One CTA waits on an mbarrier that nothing arrives on.  The bounded wait
// gives up after timeout_ns, records the timeout and the kernel returns.
__global__ void wait_timeout_probe_kernel(unsigned* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait(smem_u32(&bar), 0, &abort_flag, err, timeout_ns);
  }
  __syncthreads();
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_last_device_error(void) {
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    (void)cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  unsigned w = 0;
  if (cudaMemcpy(&w, d->err_word, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpy(d->err_word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (w != 0 && clear_gemm_scratch(d->device) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (w == kErrTimeout) return NVFP4_ERR_TIMEOUT;
  if (w != 0) return NVFP4_ERR_DEVICE;
  return NVFP4_OK;
}

void nvfp4_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns, std::memory_order_relaxed); }

int nvfp4_bounds_checked(void) { return NVFP4_BOUNDS_CHECK ? 1 : 0; }

void nvfp4_set_decode_cooperative(int enable) { g_decode_coop.store(enable ? 1 : 0, std::memory_order_relaxed); }

nvfp4_status nvfp4_test_wait_timeout(uint64_t timeout_ns, nvfp4_stream_t stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(d->err_word, timeout_ns);
  return cuda_status(cudaGetLastError());
}

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported device or size";
    case NVFP4_ERR_CUDA: return "CUDA runtime or launch failure";
    case NVFP4_ERR_TIMEOUT: return "a kernel wait timed out";
    case NVFP4_ERR_DEVICE: return "a kernel detected an out-of-range index";
  }
  return "unknown status";
}

int nvfp4_version(void) { return 100; }

}  // extern "C"
