// Per-block NVFP4 quantization arithmetic shared by the quantize kernel and
// the GEMM that quantizes its activation operand itself.  Both must encode
// bit for bit alike, so both call quantize_block().
//
// Format [picx.dev summary of "Why Gated DeltaNet Survives 4-Bit
// Quantization", "Background"]: E2M1 values, one E4M3 scale per 16-element
// block set from blockmax/6, one FP32 scale per tensor.  Per block:
//   amax_b = max|x|, t = (amax_b/6)*g, s = E4M3_rn_sat(t),
//   s == 0 -> signed-zero codes, else r = g/e4m3(s), code = E2M1_rn_sat(x*r).
// All FP32 steps use explicitly rounded intrinsics (no contraction), and the
// FP8/FP4 encodings use the hardware cvt.rn.satfinite conversions.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace nvfp4 {

// Unsigned division by an invariant divisor d (Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994, unsigned
// case): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// n / d == (mulhi(n, m) + n) >> l for every 32-bit n.
struct DivU32 {
  uint32_t m, l;
};

__device__ __forceinline__ uint32_t div_u32(uint32_t n, DivU32 d) {
  const uint32_t t = __umulhi(n, d.m);
  return (uint32_t)(((uint64_t)t + n) >> d.l);
}

// Host side: the (m, l) pair for divisor d >= 1.
inline DivU32 make_div(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  DivU32 r;
  r.l = l;
  r.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
  return r;
}


// ----------------------------------------------------------------- encoders

__device__ __forceinline__ uint32_t cvt_e4m3(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(t), "f"(t));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t s) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(s & 0xFF);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// Eight floats -> eight E2M1 codes, element 0 in the low nibble of the low byte.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&y)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.u32.u8 %0, b0;\n\t}"
      : "=r"(out)
      : "f"(lo), "f"(hi));
  return out;
}

// One thread owns one 16-element block: 32 (bf16) or 64 (f32) contiguous
// bytes in, 8 bytes of codes and one scale byte out; a warp reads 1 KB
// (bf16) and writes 256 contiguous bytes of codes.
template <bool kF32>
struct Block16 {
  uint4 v[kF32 ? 4 : 2];
};

// The 16 elements at p (16-byte aligned), through the L1/L2 read-only path
// (for data that several CTAs read).
template <bool kF32>
__device__ __forceinline__ void load_block_at(const void* p, Block16<kF32>& B) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < (kF32 ? 4 : 2); ++i) B.v[i] = __ldg(q + i);
}

template <bool kF32>
__device__ __forceinline__ void load_block(const void* x, uint32_t b, Block16<kF32>& B) {
  const uint4* p = reinterpret_cast<const uint4*>(x) + (size_t)b * (kF32 ? 4 : 2);
#pragma unroll
  for (int i = 0; i < (kF32 ? 4 : 2); ++i) B.v[i] = __ldcs(p + i);
}

// Largest magnitude of the block.  bf16: clear both sign bits of each packed
// pair and take the unsigned 16-bit maximum (non-negative bf16 bit patterns
// order like their values; inputs are finite), then widen exactly to f32.
template <bool kF32>
__device__ __forceinline__ float block_amax(const Block16<kF32>& B) {
  if constexpr (kF32) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m = fmaxf(m, fabsf(__uint_as_float(B.v[i].x)));
      m = fmaxf(m, fabsf(__uint_as_float(B.v[i].y)));
      m = fmaxf(m, fabsf(__uint_as_float(B.v[i].z)));
      m = fmaxf(m, fabsf(__uint_as_float(B.v[i].w)));
    }
    return m;
  } else {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      w = __vmaxu2(w, B.v[i].x & 0x7FFF7FFFu);
      w = __vmaxu2(w, B.v[i].y & 0x7FFF7FFFu);
      w = __vmaxu2(w, B.v[i].z & 0x7FFF7FFFu);
      w = __vmaxu2(w, B.v[i].w & 0x7FFF7FFFu);
    }
    const uint32_t m16 = max(w >> 16, w & 0xFFFFu);
    return __uint_as_float(m16 << 16);
  }
}

template <bool kF32>
__device__ __forceinline__ void block_floats(const Block16<kF32>& B, float (&f)[16]) {
  if constexpr (kF32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[4 * i + 0] = __uint_as_float(B.v[i].x);
      f[4 * i + 1] = __uint_as_float(B.v[i].y);
      f[4 * i + 2] = __uint_as_float(B.v[i].z);
      f[4 * i + 3] = __uint_as_float(B.v[i].w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t w[4] = {B.v[i].x, B.v[i].y, B.v[i].z, B.v[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[8 * i + 2 * k] = __uint_as_float(w[k] << 16);              // bf16 -> f32 is exact
        f[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  }
}

// rtab entry for scale byte s: g / e4m3(s) for s in 1..126, 0 otherwise.
__device__ __forceinline__ float recip_entry(float g, uint32_t s) {
  return (s >= 1 && s <= 126) ? __fdiv_rn(g, e4m3_to_f32(s)) : 0.0f;
}

// One 16-element block: returns the scale byte and the 16 codes (lo: elements
// 0-7, hi: elements 8-15, element 0 in the low nibble).  rtab as above.
template <bool kF32>
__device__ __forceinline__ uint32_t quantize_block(const Block16<kF32>& B, float g, const float* rtab,
                                                   uint32_t& lo, uint32_t& hi, float* amax_out = nullptr) {
  const float amax = block_amax<kF32>(B);
  if (amax_out) *amax_out = amax;
  const float q = __fdiv_rn(amax, 6.0f);
  const float t = __fmul_rn(q, g);
  const uint32_t s = cvt_e4m3(t);
  float f[16];
  block_floats<kF32>(B, f);
  if (s == 0) {
    lo = hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo |= ((__float_as_uint(f[i]) >> 31) << 3) << (4 * i);
      hi |= ((__float_as_uint(f[8 + i]) >> 31) << 3) << (4 * i);
    }
  } else {
    const float r = rtab[s];
    float y0[8], y1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      y0[i] = __fmul_rn(f[i], r);
      y1[i] = __fmul_rn(f[8 + i], r);
    }
    lo = cvt_e2m1x8(y0);
    hi = cvt_e2m1x8(y1);
  }
  return s;
}

}  // namespace nvfp4
