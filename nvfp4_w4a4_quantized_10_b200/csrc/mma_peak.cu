// Dense FP4 tensor-core throughput of the device, measured rather than
// quoted: every SM issues back-to-back block-scaled FP4 MMAs of the shape the
// prefill GEMM issues (tcgen05.mma kind::mxf4nvf4, M = 128, N = 256, K = 64,
// E4M3 scales for 16-element blocks) from operands resident in shared memory,
// so no memory traffic limits it.  The figure is the denominator a
// tensor-bound kernel of this library can be held against, next to the
// nominal dense FP4 rate and the measured BF16 rate times the nominal
// FP4 : BF16 ratio.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "common.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kPeakOffA = 0;            // 128 rows x 128 B (four K = 64 blocks)
constexpr int kPeakOffB = 16384;        // 256 rows x 128 B
constexpr int kPeakOffSf = 49152;       // 3 x 4 scale chunks of 512 B (A, B rows 0-127, B rows 128-255)
constexpr int kPeakOffBar = kPeakOffSf + 12 * 512;
constexpr int kPeakSmem = kPeakOffBar + 64 + 1024;   // + alignment slack
constexpr int kPeakThreads = 128;
constexpr int kPeakMaxCtas = 1024;

// per-CTA cycle counts of the timed launch (no allocation in the library)
__device__ unsigned long long g_peak_cycles[kPeakMaxCtas];

__global__ void __launch_bounds__(kPeakThreads, 1)
    mma_peak_kernel(int iters, unsigned* err, uint64_t timeout_ns, uint64_t drain_ns, unsigned long long* cycles) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  // operands: any nibble is a valid E2M1 code; scale bytes 0x30-0x3F are
  // finite E4M3 values near 1
  for (int i = threadIdx.x; i < kPeakOffBar / 4; i += blockDim.x) {
    uint32_t v = (uint32_t)i * 2654435761u;
    if (i * 4 >= kPeakOffSf) v = 0x38383838u ^ (v & 0x07070707u);
    reinterpret_cast<uint32_t*>(smem)[i] = v;
  }
  const uint32_t bar = sb + kPeakOffBar;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);        // the MMAs have completed
    mbar_init(bar + 8, 1);    // the scale copies have landed
    mbar_init(bar + 16, 1);   // drain before TMEM is freed
    abort_flag = 0;
    fence_barrier_init();
  }
  fence_proxy_async_smem();           // generic-proxy writes -> tensor-core reads
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(&tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_holder;
  if (threadIdx.x == 0) {
    // accumulator in columns [0, 256); A scales at 256 (4 columns per K
    // block), B scales at 272 (8 columns per K block: two 128-row blocks)
    const uint32_t sfa = tm + 256, sfb = tm + 272;
    const uint64_t sdesc = smem_desc(sb + kPeakOffSf, 16, 128, 0);
    for (int kb = 0; kb < 4; ++kb) {
      tc_cp_32x128b_warpx4(sfa + kb * 4, sdesc + (uint64_t)(kb * 32));
      for (int rb = 0; rb < 2; ++rb)
        tc_cp_32x128b_warpx4(sfb + kb * 8 + rb * 4, sdesc + (uint64_t)(((1 + rb) * 4 + kb) * 32));
    }
    const uint64_t ad = smem_desc(sb + kPeakOffA, 16, 1024, 2);
    const uint64_t bd = smem_desc(sb + kPeakOffB, 16, 1024, 2);
    constexpr uint32_t idesc = idesc_nvf4(128, 256);
    tc_commit(bar + 8);                // the scale copies have landed before the clock starts
    if (mbar_wait(bar + 8, 0, &abort_flag, err, timeout_ns)) {
      tc_fence_after();
      const long long t0 = clock64();
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          tc_mma_block_scaled<false>(tm, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2), idesc, sfa + kb * 4,
                                     sfb + kb * 8, (it | kb) != 0 ? 1u : 0u);
      }
      tc_commit(bar);
      const bool ok = mbar_wait(bar, 0, &abort_flag, err, timeout_ns);
      const long long t1 = clock64();
      cycles[blockIdx.x] = ok ? (unsigned long long)(t1 - t0) : 0ull;
    } else {
      cycles[blockIdx.x] = 0ull;
    }
    // every tensor-core operation of this thread has completed before TMEM
    // is freed, whichever wait above gave up
    volatile int never = 0;
    tc_commit(bar + 16);
    (void)mbar_wait(bar + 16, 0, &never, err, drain_ns);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tm, 512);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_measure_mma_peak(int iters, double* tflops, double* flop_per_clk_per_sm, nvfp4_stream_t stream) {
  if (iters < 1 || iters > (1 << 20) || !tflops || !flop_per_clk_per_sm) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (d->major != 10) return NVFP4_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPeakSmem);
  if (e != cudaSuccess) return cuda_status(e);
  const int grid = d->sm_count;
  if (grid > kPeakMaxCtas) return NVFP4_ERR_UNSUPPORTED;
  void* cyc_addr = nullptr;
  e = cudaGetSymbolAddress(&cyc_addr, g_peak_cycles);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned long long* cyc = static_cast<unsigned long long*>(cyc_addr);
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  nvfp4_status status = NVFP4_OK;
  float ms = 0.f;
  std::vector<unsigned long long> h(grid);
  if (cudaEventCreate(&ev0) != cudaSuccess || cudaEventCreate(&ev1) != cudaSuccess) {
    status = NVFP4_ERR_CUDA;
  } else {
    const uint64_t to = wait_timeout_ns(), dr = drain_timeout_ns();
    mma_peak_kernel<<<grid, kPeakThreads, kPeakSmem, st>>>(iters, d->err_word, to, dr, cyc);   // warm-up
    cudaEventRecord(ev0, st);
    mma_peak_kernel<<<grid, kPeakThreads, kPeakSmem, st>>>(iters, d->err_word, to, dr, cyc);
    cudaEventRecord(ev1, st);
    if (cudaEventSynchronize(ev1) != cudaSuccess || cudaEventElapsedTime(&ms, ev0, ev1) != cudaSuccess ||
        cudaMemcpy(h.data(), cyc, sizeof(unsigned long long) * grid, cudaMemcpyDeviceToHost) != cudaSuccess)
      status = NVFP4_ERR_CUDA;
  }
  if (ev0) cudaEventDestroy(ev0);
  if (ev1) cudaEventDestroy(ev1);
  if (status != NVFP4_OK) {
    (void)cudaGetLastError();
    return status;
  }
  const double flop_per_cta = 2.0 * 128 * 256 * 64 * 4 * (double)iters;
  std::sort(h.begin(), h.end());
  const unsigned long long med = h[grid / 2];
  if (med == 0 || ms <= 0.f) return NVFP4_ERR_TIMEOUT;
  *tflops = flop_per_cta * grid / (ms * 1e-3) / 1e12;
  *flop_per_clk_per_sm = flop_per_cta / (double)med;
  return NVFP4_OK;
}

}  // extern "C"
