// NVFP4 activation quantization, per-tensor amax, scale-layout rewrite and
// the element conversions.  The per-block arithmetic (and its citation) is in
// block_quant.cuh, shared with the GEMM that quantizes its own activation.
//
// Work split: one thread owns one 16-element block (two 16-byte loads for
// bf16), so the per-block scalar work (two FP32 roundings, the E4M3
// conversion, the scale store) is done once per 16 elements; a warp reads
// 1 KB and writes 256 contiguous bytes of codes.  The kernel is meant to be
// HBM-bound (2.5625 bytes per bf16 element); each thread loads two blocks
// (four 16-byte loads in flight) and the grid covers the tensor in one pass,
// so the hardware block scheduler keeps every SM fed until the tail instead
// of a persistent grid whose threads walk the tensor in lock step.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "block_quant.cuh"
#include "common.h"
#include "ptx.cuh"

namespace nvfp4 {

// Offset of scale j of row r in the tensor-core scale layout.
__device__ __forceinline__ int64_t tc_scale_offset(int64_t r, int64_t j, int64_t kc) {
  return ((r >> 7) * kc + (j >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// Raise *amax to v.  Non-negative floats order like their bit patterns, so
// an unsigned atomic maximum does it; the word only grows while the kernel
// runs, so a CTA whose maximum is not above a value it reads there has
// nothing to add and skips the atomic (most CTAs, after the first few).
__device__ __forceinline__ void update_amax(float* amax, float v) {
  unsigned* w = reinterpret_cast<unsigned*>(amax);
  const unsigned bits = __float_as_uint(v);
  if (bits > __ldcg(w)) atomicMax(w, bits);
}

// amax_out = 0 in stream order: launched as a programmatic dependent (it
// waits for the previous kernel before the store), and the amax kernel after
// it waits for it in turn.  Keeps the dependent-launch chain that a memset
// node would break.
__global__ void zero_word_kernel(float* p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) *p = 0.0f;
}

// Grid-stride over 16-element blocks.  Blocks of rows [M, rows_total) exist
// only in the tensor-core layout (rows padded to 128): they read nothing and
// write zero scales.  rtab[s] = g / e4m3(s) for every scale byte, computed
// once per CTA with the same correctly rounded division the block formula
// uses.
template <bool kF32, bool kTC, bool kAmax>
__global__ void __launch_bounds__(256) quantize_kernel(const void* __restrict__ x, uint32_t real_blocks,
                                                       uint32_t total_blocks, uint32_t nblk, DivU32 div_nblk,
                                                       float g, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales, float* amax_out,
                                                       int64_t kc, uint64_t codes_bytes, uint64_t scale_bytes,
                                                       unsigned* err) {
  constexpr int U = 2;
  // programmatic dependent launch: let the next kernel (the GEMM) start its
  // prologue and weight loads now, and wait until the previous kernel in the
  // stream has completed before touching memory it may read or write
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float rtab[256];
  {
    const uint32_t s = threadIdx.x;
    rtab[s] = recip_entry(g, s);
  }
  __syncthreads();
  const uint32_t stride = gridDim.x * blockDim.x;
  float local_max = 0.0f;

  for (uint32_t base = blockIdx.x * blockDim.x + threadIdx.x; base < total_blocks; base += U * stride) {
    Block16<kF32> B[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t b = base + u * stride;
      if (b < real_blocks) load_block<kF32>(x, b, B[u]);
      else {
#pragma unroll
        for (int i = 0; i < (kF32 ? 4 : 2); ++i) B[u].v[i] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t b = base + u * stride;
      if (b >= total_blocks) break;
      uint32_t lo, hi;
      float amax;
      const uint32_t s = quantize_block<kF32>(B[u], g, rtab, lo, hi, &amax);
      if constexpr (kAmax) local_max = fmaxf(local_max, amax);
      if (b < real_blocks && bounds_ok((uint64_t)(b + 1) * 8 <= codes_bytes, err))
        reinterpret_cast<uint2*>(codes)[b] = make_uint2(lo, hi);
      if constexpr (kTC) {
        const uint32_t row = div_u32(b, div_nblk);
        const uint32_t j = b - row * nblk;
        const int64_t o = tc_scale_offset(row, j, kc);
        if (bounds_ok((uint64_t)o < scale_bytes, err)) scales[o] = (uint8_t)s;
        // K % 64 == 32: the last chunk of the row has two padding slots
        if (j == nblk - 1 && (nblk & 3) == 2) {
          const int64_t o1 = tc_scale_offset(row, j + 1, kc), o2 = tc_scale_offset(row, j + 2, kc);
          if (bounds_ok((uint64_t)o1 < scale_bytes && (uint64_t)o2 < scale_bytes, err)) {
            scales[o1] = 0;
            scales[o2] = 0;
          }
        }
      } else {
        if (bounds_ok((uint64_t)b < scale_bytes, err)) scales[b] = (uint8_t)s;
      }
    }
  }

  if constexpr (kAmax) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local_max = fmaxf(local_max, __shfl_xor_sync(0xFFFFFFFFu, local_max, o));
    __shared__ float wmax[8];
    if (lane == 0) wmax[threadIdx.x >> 5] = local_max;
    __syncthreads();
    if (threadIdx.x == 0) {
      float bmax = 0.0f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) bmax = fmaxf(bmax, wmax[w]);
      update_amax(amax_out, bmax);
    }
  }
}

template <bool kF32>
__device__ __forceinline__ float vec_absmax(const uint4& v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (kF32) {
      m = fmaxf(m, fabsf(__uint_as_float(w[k])));
    } else {
      m = fmaxf(m, fabsf(__uint_as_float(w[k] << 16)));
      m = fmaxf(m, fabsf(__uint_as_float(w[k] & 0xFFFF0000u)));
    }
  }
  return m;
}

template <bool kF32>
__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ x, int64_t n_vec, float* amax_out) {
  // n_vec 16-byte vectors; any tail elements are handled by the host-chosen
  // element count being a multiple of the vector width (K*M*elt % 16 == 0).
  // Launched as a programmatic dependent: the next kernel may start its
  // prologue now; x is read only after the previous kernel has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float m = 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + stride < n_vec; i += 2 * stride) {  // two loads in flight per thread
    const uint4 a = __ldcs(xv + i);
    const uint4 b = __ldcs(xv + i + stride);
    m = vec_absmax<kF32>(b, vec_absmax<kF32>(a, m));
  }
  if (i < n_vec) m = vec_absmax<kF32>(__ldcs(xv + i), m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = fmaxf(b, wmax[w]);
    update_amax(amax_out, b);
  }
}

// One thread per 4-byte word of the tensor-core layout.
__global__ void swizzle_scales_kernel(const uint8_t* __restrict__ rm, int64_t R, int64_t nblk, int64_t kc,
                                      int64_t n_words, uint32_t* __restrict__ tc) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_words; w += stride) {
    const int64_t chunk = w >> 7;
    const int64_t o = (w & 127) * 4;
    const int64_t rb = chunk / kc, cb = chunk - rb * kc;
    const int64_t row = rb * 128 + (o >> 4) + 32 * ((o & 15) >> 2);
    uint32_t word = 0;
    if (row < R) {
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int64_t j = cb * 4 + t;
        if (j < nblk) word |= (uint32_t)rm[row * nblk + j] << (8 * t);
      }
    }
    tc[w] = word;
  }
}

__global__ void convert_e4m3_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = (uint8_t)cvt_e4m3(in[i]);
}

__global__ void convert_e2m1_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, int64_t n_pairs) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_pairs; j += stride)
    out[j] = (uint8_t)cvt_e2m1x2(in[2 * j], in[2 * j + 1]);
}

namespace {

int grid_for(int64_t work_items, int threads, const DeviceInfo* d, int per_sm = 8) {
  int64_t blocks = ceil_div(work_items, threads);
  const int64_t cap = (int64_t)d->sm_count * per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}


template <bool kF32, bool kTC, bool kAmax>
cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, float g, uint8_t* codes, uint8_t* scales,
                            float* amax_out, cudaStream_t st, const DeviceInfo* d) {
  const int64_t rows_total = kTC ? ceil_div(M, 128) * 128 : M;
  const int64_t kc = ceil_div(K, 64);
  const uint32_t nblk = (uint32_t)(K / 16);
  const uint32_t real = (uint32_t)(M * (K / 16));
  const uint32_t total = (uint32_t)(rows_total * (K / 16));
  // 256 threads, 2 blocks of 16 elements per thread, one pass over the
  // tensor (no persistent cap): with L2-cold inputs this ran 4096x5120,
  // 4096x17408 and 32768x5120 bf16 at 0.76, 0.89 and 0.95 of the measured
  // copy bandwidth, against 0.74, 0.83 and 0.87 for a persistent grid of 4
  // CTAs per SM walking the tensor in two-block steps
  const int threads = 256;
  const int blocks = grid_for(ceil_div(total, 2), threads, d, 1 << 20);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint64_t codes_bytes = (uint64_t)M * (uint64_t)(K / 2);
  const uint64_t scale_bytes = kTC ? (uint64_t)(rows_total / 128) * kc * 512 : (uint64_t)M * (uint64_t)(K / 16);
  return cudaLaunchKernelEx(&cfg, quantize_kernel<kF32, kTC, kAmax>, x, real, total, nblk, make_div(nblk), g, codes,
                            scales, amax_out, kc, codes_bytes, scale_bytes, d->err_word);
}

cudaError_t launch_amax(const void* x, bool f32, int64_t n_vec, float* amax_out, cudaStream_t st,
                        const DeviceInfo* d) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_for(ceil_div(n_vec, 2), 256, d, 8));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return f32 ? cudaLaunchKernelEx(&cfg, amax_kernel<true>, x, n_vec, amax_out)
             : cudaLaunchKernelEx(&cfg, amax_kernel<false>, x, n_vec, amax_out);
}

cudaError_t launch_zero_word(float* p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, zero_word_kernel, p);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_scale_bytes(int64_t rows, int64_t K, nvfp4_sf_layout layout) {
  if (rows < 1 || K < 16 || K % 16 != 0) return 0;
  if (layout == NVFP4_SF_ROWMAJOR) return (size_t)(rows * (K / 16));
  if (layout == NVFP4_SF_TCGEN05) return (size_t)(ceil_div(rows, 128) * ceil_div(K, 64) * 512);
  return 0;
}

nvfp4_status nvfp4_amax(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K, float* amax_out,
                        nvfp4_stream_t stream) {
  if (!x || !amax_out || M < 1 || K < 1) return NVFP4_ERR_INVALID_ARG;
  if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  const int64_t elt = dtype == NVFP4_IN_F32 ? 4 : 2;
  if ((M * K * elt) % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(amax_out) & 3)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = launch_zero_word(amax_out, st);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_amax(x, dtype == NVFP4_IN_F32, M * K * elt / 16, amax_out, st, d));
}

nvfp4_status nvfp4_amax_accumulate(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K,
                                   float* running_amax, nvfp4_stream_t stream) {
  if (!x || !running_amax || M < 1 || K < 1) return NVFP4_ERR_INVALID_ARG;
  if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  const int64_t elt = dtype == NVFP4_IN_F32 ? 4 : 2;
  if ((M * K * elt) % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(running_amax) & 3)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  return cuda_status(launch_amax(x, dtype == NVFP4_IN_F32, M * K * elt / 16, running_amax,
                                 (cudaStream_t)stream, d));
}

nvfp4_status nvfp4_quantize(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K, float global_scale,
                            uint8_t* codes, uint8_t* block_scales, nvfp4_sf_layout layout, float* amax_out,
                            nvfp4_stream_t stream) {
  if (!x || !codes || !block_scales || M < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  if (ceil_div(M, 128) * 128 * (K / 16) >= (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(global_scale)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(block_scales)) return NVFP4_ERR_ALIGNMENT;
  if (amax_out && (reinterpret_cast<uintptr_t>(amax_out) & 3)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (amax_out) {
    cudaError_t e = launch_zero_word(amax_out, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  const bool f32 = dtype == NVFP4_IN_F32, tc = layout == NVFP4_SF_TCGEN05, am = amax_out != nullptr;
  cudaError_t e;
#define NVFP4_Q(A, B, C) \
  if (f32 == A && tc == B && am == C) e = launch_quantize<A, B, C>(x, M, K, global_scale, codes, block_scales, amax_out, st, d);
  NVFP4_Q(false, false, false) else NVFP4_Q(false, false, true) else NVFP4_Q(false, true, false)
  else NVFP4_Q(false, true, true) else NVFP4_Q(true, false, false) else NVFP4_Q(true, false, true)
  else NVFP4_Q(true, true, false) else NVFP4_Q(true, true, true) else e = cudaErrorInvalidValue;
#undef NVFP4_Q
  return cuda_status(e);
}

nvfp4_status nvfp4_test_bounds_check(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* block_scales,
                                     nvfp4_stream_t stream) {
  if (!NVFP4_BOUNDS_CHECK) return NVFP4_ERR_UNSUPPORTED;   // the release build has no checks to exercise
  if (!x || !codes || !block_scales || M < 1 || K < 64 || K % 64 != 0) return NVFP4_ERR_INVALID_ARG;
  if (ceil_div(M, 128) * 128 * (K / 16) >= (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(block_scales)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  // the quantizer, told that the scale buffer ends one 512-byte chunk early:
  // the scales of the last chunk fail the check (their real addresses are
  // inside the caller's full-size buffer, so nothing out of range is touched)
  const int64_t rows_total = ceil_div(M, 128) * 128, kc = K / 64;
  const uint32_t nblk = (uint32_t)(K / 16);
  const uint32_t real = (uint32_t)(M * (K / 16)), total = (uint32_t)(rows_total * (K / 16));
  const uint64_t codes_bytes = (uint64_t)M * (uint64_t)(K / 2);
  const uint64_t short_scales = (uint64_t)(rows_total / 128) * kc * 512 - 512;
  const int blocks = grid_for(ceil_div(total, 2), 256, d, 1 << 20);
  quantize_kernel<false, true, false><<<blocks, 256, 0, (cudaStream_t)stream>>>(
      x, real, total, nblk, make_div(nblk), 1.0f, codes, block_scales, nullptr, kc, codes_bytes, short_scales,
      d->err_word);
  return cuda_status(cudaGetLastError());
}

nvfp4_status nvfp4_swizzle_scales(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* tc,
                                  nvfp4_stream_t stream) {
  if (!rowmajor || !tc || rows < 1 || K < 16 || K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(tc)) return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  const int64_t kc = ceil_div(K, 64);
  const int64_t n_words = ceil_div(rows, 128) * kc * 128;
  const int blocks = grid_for(n_words, 256, d, 8);
  swizzle_scales_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(rowmajor, rows, K / 16, kc, n_words,
                                                                  reinterpret_cast<uint32_t*>(tc));
  return cuda_status(cudaGetLastError());
}

nvfp4_status nvfp4_convert_e4m3(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream) {
  if (!in || !out || n < 1) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  convert_e4m3_kernel<<<grid_for(n, 256, d, 8), 256, 0, (cudaStream_t)stream>>>(in, out, n);
  return cuda_status(cudaGetLastError());
}

nvfp4_status nvfp4_convert_e2m1(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream) {
  if (!in || !out || n < 2 || (n & 1)) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  convert_e2m1_kernel<<<grid_for(n / 2, 256, d, 8), 256, 0, (cudaStream_t)stream>>>(in, out, n / 2);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
