// Host-side helpers shared by the library's translation units: argument
// checks, per-device state (error word, SM count, architecture), launch
// configuration.  No torch types; plain CUDA runtime.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/nvfp4.h"

namespace nvfp4 {

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int major = 0, minor = 0;
  size_t max_smem_optin = 0;
  unsigned* err_word = nullptr;  // device address of this device's error word
};

// Per-device information; initialised on first use on the current device.
// Returns nullptr if the CUDA runtime fails.
const DeviceInfo* device_info();

// Wait bound for every kernel of the library (ns).
uint64_t wait_timeout_ns();

// Bound on a CTA's waits for its own in-flight copies and tensor-core work
// before it frees shared memory and TMEM and exits: at least 1 s whatever the
// wait bound above, so that a short wait bound (a test, or a caller that
// wants quick failure reports) never lets a CTA exit under live copies.
uint64_t drain_timeout_ns();

// Whether split-K (decode) GEMM grids launch as cooperative grids, which the
// driver admits only when every CTA can be resident at once.
bool decode_cooperative();

// Empties every K-split scratch buffer of the GEMM on `device` (after a
// device-side error left partial words behind).  Synchronous.
cudaError_t clear_gemm_scratch(int device);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool finite_positive(float g) {
  uint32_t b;
  std::memcpy(&b, &g, 4);
  const bool finite = ((b >> 23) & 0xFF) != 0xFF;
  return finite && g > 0.0f;
}

inline nvfp4_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  (void)cudaGetLastError();  // do not leave a sticky launch error for the caller's next check
  // a cooperative (co-residency guaranteed) grid that cannot be resident at once
  if (e == cudaErrorCooperativeLaunchTooLarge) return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_ERR_CUDA;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace nvfp4
