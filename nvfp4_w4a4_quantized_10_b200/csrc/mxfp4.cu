// MXFP4 quantization, the contrast format: 32-element blocks sharing one
// power-of-two (E8M0) scale, where NVFP4 uses 16-element blocks with an E4M3
// scale and a per-tensor FP32 scale [anthology record LIT-800, "Standing in
// the anthology"].  The conversion is the published OCP Microscaling v1.0
// rule for MXFP4: per block of 32 along K,
//     E = floor(log2(max |x|)) - 2,  clamped to [-127, 127]
// (2 = exponent of E2M1's largest normal, 6 = 1.5 * 2^2); the scale byte is
// E + 127 and each code is E2M1(x * 2^-E), nearest even, saturating at 6.
// An all-zero block gets byte 0.  floor(log2(amax)) is amax's exponent field
// minus the bias, and the clamp at -127 covers subnormal and zero maxima, so
// the byte is max(exponent field - 2, 0); x * 2^-E is a power-of-two scaling
// (exact unless the product is an FP32 subnormal, whose code is a signed zero
// either way).
//
// Work split: two threads per 32-element block, each owning 16 elements (the
// NVFP4 quantizer's access pattern: two 16-byte loads of bf16 per thread, a
// warp reads 1 KB); the pair combines its maxima with one shuffle.  Each
// thread keeps two such items in flight per iteration.  HBM-bound:
// 2 + 0.5 + 1/32 bytes per bf16 element.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "block_quant.cuh"
#include "common.h"
#include "ptx.cuh"

namespace nvfp4 {

// Work item t (whole warps step together, so both threads of a pair are
// always present for the shuffle): block p = t / 2, half h = t % 2, row
// r = p / nblk_pad, block column j = p % nblk_pad.  In the TCGEN05 layout rows
// are padded to 128 and block columns to a multiple of 4; padding slots only
// write a zero scale byte.
template <bool kF32, bool kTC>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const void* __restrict__ x, int64_t M, int64_t K,
                                                          int64_t nblk_pad, DivU32 div_nblk_pad, int64_t total_items,
                                                          uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ scales, int64_t kc,
                                                          uint64_t codes_bytes, uint64_t scale_bytes, unsigned* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t nblk = K / 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // two work items per thread per iteration, both loads issued first
  for (int64_t wb = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); wb < total_items; wb += 2 * stride) {
    Block16<kF32> B[2];
    bool real[2], live[2];
    int64_t r[2], j[2];
    int h[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t t = wb + u * stride + lane;
      live[u] = t < total_items;
      const int64_t pb = t >> 1;
      h[u] = (int)(t & 1);
      r[u] = div_u32((uint32_t)pb, div_nblk_pad);   // pb < 2^31 (checked on the host)
      j[u] = pb - r[u] * nblk_pad;
      real[u] = live[u] && r[u] < M && j[u] < nblk;
      if (real[u]) load_block<kF32>(x, (uint32_t)(r[u] * (K / 16) + 2 * j[u] + h[u]), B[u]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (wb + u * stride >= total_items) break;          // warp-uniform
      float f[16];
      float amax = 0.0f;
      if (real[u]) {
        amax = block_amax<kF32>(B[u]);
        block_floats<kF32>(B[u], f);
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      if (!live[u]) continue;
      const uint32_t ef = __float_as_uint(amax) >> 23;        // amax >= 0: the exponent field
      const uint32_t sbyte = ef >= 2 ? ef - 2 : 0;             // E + 127
      if (real[u]) {
        const float inv = __uint_as_float((254u - sbyte) << 23);  // 2^-E, normal for every byte produced
        float lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          lo[i] = f[i] * inv;
          hi[i] = f[8 + i] * inv;
        }
        const int64_t co = r[u] * (K / 2) + j[u] * 16 + h[u] * 8;
        if (bounds_ok((uint64_t)co + 8 <= codes_bytes, err))
          *reinterpret_cast<uint2*>(codes + co) = make_uint2(cvt_e2m1x8(lo), cvt_e2m1x8(hi));
      }
      if (h[u] == 0) {
        const int64_t off = kTC ? ((r[u] >> 7) * kc + (j[u] >> 2)) * 512 + (r[u] & 31) * 16 + ((r[u] >> 5) & 3) * 4 +
                                      (j[u] & 3)
                                : r[u] * nblk + j[u];
        if (bounds_ok((uint64_t)off < scale_bytes, err)) scales[off] = real[u] ? (uint8_t)sbyte : (uint8_t)0;
      }
    }
  }
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K, uint8_t* codes,
                               uint8_t* scales, nvfp4_sf_layout layout, nvfp4_stream_t stream) {
  if (!x || !codes || !scales || M < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (ceil_div(M, 128) * 128 * (K / 16) >= (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  const bool tc = layout == NVFP4_SF_TCGEN05;
  const int64_t kc = ceil_div(K, 128);
  const int64_t rows = tc ? ceil_div(M, 128) * 128 : M;
  const int64_t nblk_pad = tc ? 4 * kc : K / 32;
  const int64_t total = rows * nblk_pad * 2;
  // one pass over the tensor, two items per thread (L2-cold 4096x5120 bf16:
  // 13.4 us against 15.3 us for a persistent grid of 4 CTAs per SM)
  const int blocks = (int)std::max<int64_t>(1, ceil_div(total, 512));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const bool f32 = dtype == NVFP4_IN_F32;
  const DivU32 div_np = make_div((uint32_t)nblk_pad);
  const uint64_t codes_bytes = (uint64_t)M * (uint64_t)(K / 2);
  const uint64_t scale_bytes = tc ? (uint64_t)(rows / 128) * kc * 512 : (uint64_t)M * (uint64_t)(K / 32);
  cudaError_t e;
  if (f32) e = tc ? cudaLaunchKernelEx(&cfg, mx_quantize_kernel<true, true>, x, M, K, nblk_pad, div_np, total, codes, scales, kc, codes_bytes, scale_bytes, d->err_word)
                  : cudaLaunchKernelEx(&cfg, mx_quantize_kernel<true, false>, x, M, K, nblk_pad, div_np, total, codes, scales, kc, codes_bytes, scale_bytes, d->err_word);
  else e = tc ? cudaLaunchKernelEx(&cfg, mx_quantize_kernel<false, true>, x, M, K, nblk_pad, div_np, total, codes, scales, kc, codes_bytes, scale_bytes, d->err_word)
              : cudaLaunchKernelEx(&cfg, mx_quantize_kernel<false, false>, x, M, K, nblk_pad, div_np, total, codes, scales, kc, codes_bytes, scale_bytes, d->err_word);
  return cuda_status(e);
}

}  // extern "C"
