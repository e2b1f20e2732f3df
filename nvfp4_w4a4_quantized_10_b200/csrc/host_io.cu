// The linear layer with a host-resident activation and result: one call
// enqueues, on one stream, the host-to-device copy of X, the layer itself
// (nvfp4_linear: quantize X, block-scaled GEMM, dequantizing epilogue) and
// the device-to-host copy of the output.  Host code only; the device work is
// the library's kernels.  One cudaMemcpyAsync per copy.
#include <cuda_runtime.h>

#include "common.h"

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_linear_host(const void* x_host, nvfp4_in_dtype x_dtype, int64_t M, int64_t K,
                               float a_global_scale, const uint8_t* w_codes, const uint8_t* w_scales,
                               float w_global_scale, int64_t N, void* out_host, nvfp4_out_dtype out_dtype,
                               void* x_dev, uint8_t* a_codes, uint8_t* a_scales, void* out_dev,
                               nvfp4_stream_t stream) {
  // the layer's own checks, repeated here so that a bad call enqueues nothing
  if (!x_host || !out_host || !x_dev || !out_dev || !w_codes || !w_scales) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_IN_BF16 && x_dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(a_global_scale) || !finite_positive(w_global_scale)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x_dev) || !aligned16(out_dev) || !aligned16(w_codes) || !aligned16(w_scales))
    return NVFP4_ERR_ALIGNMENT;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  const size_t x_bytes = (size_t)M * (size_t)K * (x_dtype == NVFP4_IN_F32 ? 4 : 2);
  const size_t out_bytes = (size_t)M * (size_t)N * (out_dtype == NVFP4_OUT_F32 ? 4 : 2);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_status(e);
  const nvfp4_status s = nvfp4_linear(x_dev, x_dtype, M, K, a_global_scale, w_codes, w_scales, w_global_scale, N,
                                      out_dev, out_dtype, a_codes, a_scales, stream);
  if (s != NVFP4_OK) return s;
  return cuda_status(cudaMemcpyAsync(out_host, out_dev, out_bytes, cudaMemcpyDeviceToHost, st));
}

}  // extern "C"
