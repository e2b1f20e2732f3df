// Offline global-scale harmonisation of a fused weight's block scales: the
// rows of segment i were quantized with their own global scale g_i; their
// E4M3 scales are re-encoded for one common scale g, s' = E4M3(e4m3(s) * q_i)
// with q_i = g / g_i, the element codes untouched, so that a GEMM that applies
// a single global scale serves every segment [cctest.ai article, "Main
// findings": the released checkpoint is pre-harmonized; anthology record
// LIT-800, "Standing in the anthology"].
//
// HBM-bound and run once per checkpoint: one read and one write of each
// scale byte, 16-byte vectors, grid-stride.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "block_quant.cuh"
#include "common.h"

namespace nvfp4 {

// Per-segment factors of the offline scale harmonisation: rows
// [offs[i], offs[i+1]) take q[i] = g / g_i (FP32, rounded once on the host).
struct HarmonizeSegs {
  int64_t offs[NVFP4_MAX_SEGMENTS + 1];
  float q[NVFP4_MAX_SEGMENTS];
  int n;
};

// Factor of a row's scales; -1 for a row outside every segment (or a
// TCGEN05 padding row), whose bytes are kept as they are.
__device__ __forceinline__ float segment_factor(int64_t row, const HarmonizeSegs& sg) {
  int i = 0;
  while (i < sg.n && row >= sg.offs[i + 1]) ++i;
  return i == sg.n ? -1.0f : sg.q[i];
}

// Scale bytes 0 and 1 of `pair` times their own factors, re-encoded
// (nearest-even, saturating); a byte with a negative factor is kept.
__device__ __forceinline__ uint32_t rescale_pair(uint32_t pair, float q0, float q1) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(pair & 0xFFFFu)));
  const float v0 = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))) * q0;
  const float v1 = __half2float(__ushort_as_half((unsigned short)(h2 >> 16))) * q1;
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(v1), "f"(v0));
  uint32_t out = r;
  if (q0 < 0.0f) out = (out & 0xFF00u) | (pair & 0x00FFu);
  if (q1 < 0.0f) out = (out & 0x00FFu) | (pair & 0xFF00u);
  return out;
}

__device__ __forceinline__ uint32_t rescale_word(uint32_t w, const float* f) {
  return rescale_pair(w, f[0], f[1]) | (rescale_pair(w >> 16, f[2], f[3]) << 16);
}

// One thread per 16-byte vector of the scale buffer; in may equal out (each
// thread reads its vector before writing it).  Row of byte b of vector v:
//   row-major  (16v + b) / nblk
//   TCGEN05    (chunk / kc) * 128 + (o / 16) + 32 * (b / 4),  chunk = 16v / 512,
//              o = 16v % 512  (layout: byte (r%32)*16 + ((r/32)%4)*4 + j%4 of
//              the 512-byte chunk of row block r/128 and scale column j/4),
// so a TCGEN05 word has one row and one factor.  A row-major buffer whose
// size is not a multiple of 16 ends in a partial vector, done byte by byte.
template <bool kTC>
__global__ void __launch_bounds__(256) harmonize_scales_kernel(const uint8_t* in, uint8_t* out, int64_t nblk,
                                                               int64_t kc, int64_t n_bytes, HarmonizeSegs sg) {
  // programmatic dependent launch: the next kernel may start its prologue
  // now; the scales are read only after the previous kernel has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t n_vec = (n_bytes + 15) / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n_vec; v += stride) {
    const int64_t base = v * 16;
    if (base + 16 <= n_bytes) {
      const uint4 w = *reinterpret_cast<const uint4*>(in + base);
      const uint32_t word[4] = {w.x, w.y, w.z, w.w};
      uint32_t res[4];
      if constexpr (kTC) {
        const int64_t row = ((base >> 9) / kc) * 128 + ((base & 511) >> 4);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float fq = segment_factor(row + 32 * q, sg);
          const float f[4] = {fq, fq, fq, fq};
          res[q] = rescale_word(word[q], f);
        }
      } else {
        float f[16];
        int64_t row = base / nblk, col = base - row * nblk;
        float fr = segment_factor(row, sg);
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          f[b] = fr;
          if (++col == nblk) {
            col = 0;
            fr = segment_factor(++row, sg);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) res[q] = rescale_word(word[q], f + 4 * q);
      }
      *reinterpret_cast<uint4*>(out + base) = make_uint4(res[0], res[1], res[2], res[3]);
    } else {
      // only a row-major buffer has a partial last vector
      for (int64_t i = base; i < n_bytes; ++i)
        out[i] = (uint8_t)(rescale_pair(in[i], segment_factor(i / nblk, sg), -1.0f) & 0xFFu);
    }
  }
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_harmonize_scales(const uint8_t* scales, int64_t N, int64_t K, nvfp4_sf_layout layout,
                                    const int64_t* seg_offsets, const float* seg_global_scales, int n_seg,
                                    float common_global_scale, uint8_t* out, nvfp4_stream_t stream) {
  if (!scales || !out || !seg_offsets || !seg_global_scales) return NVFP4_ERR_INVALID_ARG;
  if (N < 1 || K < 16 || K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (n_seg < 1 || n_seg > NVFP4_MAX_SEGMENTS || seg_offsets[0] != 0) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(common_global_scale)) return NVFP4_ERR_INVALID_ARG;
  HarmonizeSegs sg = {};
  sg.n = n_seg;
  for (int i = 0; i <= n_seg; ++i) {
    if (i > 0 && (seg_offsets[i] <= seg_offsets[i - 1] || seg_offsets[i] > N)) return NVFP4_ERR_INVALID_ARG;
    sg.offs[i] = seg_offsets[i];
  }
  for (int i = 0; i < n_seg; ++i) {
    if (!finite_positive(seg_global_scales[i])) return NVFP4_ERR_INVALID_ARG;
    sg.q[i] = common_global_scale / seg_global_scales[i];  // one FP32 division per segment
  }
  if (!aligned16(scales) || !aligned16(out)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  const bool tc = layout == NVFP4_SF_TCGEN05;
  const int64_t n_bytes = (int64_t)nvfp4_scale_bytes(N, K, layout);
  const int64_t kc = ceil_div(K, 64), nblk = K / 16;
  // grid-stride over 16-byte vectors, at most 8 CTAs of 256 threads per SM
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(ceil_div(n_bytes, 16), 256),
                                                                 (int64_t)d->sm_count * 8));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(tc ? cudaLaunchKernelEx(&cfg, harmonize_scales_kernel<true>, scales, out, nblk, kc, n_bytes, sg)
                        : cudaLaunchKernelEx(&cfg, harmonize_scales_kernel<false>, scales, out, nblk, kc, n_bytes,
                                             sg));
}

}  // extern "C"
