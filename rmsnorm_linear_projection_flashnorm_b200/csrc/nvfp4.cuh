// NVFP4 output encoding used by the quantising SwiGLU epilogues.
//
// The SwiGLU activation is written straight from the epilogue registers in
// the form the next (down) projection reads, as on the FlashInfer PR #4040
// analysis (silu_and_mul fused with the NVFP4 quantisation: e2m1 elements,
// one scale factor per SF_VEC_SIZE = 16 elements, a global scale).  Per row
// and block of 16 consecutive output columns, with gs the fp32 global scale:
//   amax = max |v|
//   sf   = RN_e4m3_satfinite(gs * amax / 6)       6: the largest e2m1 value
//   q    = RN_e2m1_satfinite(v * (gs / sf))        all zero when sf is zero
// A block holding a non-finite value gets the e4m3 NaN code 0x7F and zero
// codes.  Dequantised: e2m1(q) * e4m3(sf) / gs.  Two codes per byte with the
// even column in the low nibble; scale codes row-major [M, N / 16], or in the
// 128 x 4 chunked layout that block-scaled tensor-core GEMMs read (the
// "swizzled" scale factors of the PR #4040 analysis, fp4_sf_offset).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace fn {

constexpr int kFp4Block = 16;

// Byte offset of the scale of row m, block j (C = N / 16 scale columns, a
// multiple of 8): row-major, or chunked: rows in blocks of 128 and scale
// columns in groups of 4 make 512-byte chunks, chunk (m / 128, j / 4) at
// 512 * ((m / 128) * (C / 4) + j / 4), and inside a chunk row m, column j at
// 16 * (m mod 32) + 4 * ((m mod 128) / 32) + (j mod 4).
__device__ __forceinline__ int64_t fp4_sf_offset(int64_t m, int j, int C, bool chunked) {
  if (!chunked) return m * C + j;
  return 512 * ((m >> 7) * (C >> 2) + (j >> 2)) + 16 * (m & 31) + 4 * ((m & 127) >> 5) + (j & 3);
}

// The 8 scale bytes of row m, blocks j0 .. j0+7 (j0 a multiple of 8): one
// 8-byte store row-major, two 4-byte stores chunked.
__device__ __forceinline__ void fp4_store_sf8(uint8_t* ysf, int64_t m, int j0, int C, bool chunked, uint2 v) {
  if (!chunked) {
    *reinterpret_cast<uint2*>(ysf + m * C + j0) = v;
    return;
  }
  *reinterpret_cast<uint32_t*>(ysf + fp4_sf_offset(m, j0, C, true)) = v.x;
  *reinterpret_cast<uint32_t*>(ysf + fp4_sf_offset(m, j0 + 4, C, true)) = v.y;
}

// |v| as a bit pattern.  The unsigned maximum of these orders finite values by
// magnitude and ranks inf and NaN above every finite value.
__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

struct Fp4Scale {
  uint32_t code;   // e4m3 scale byte
  float enc;       // gs / sf: the multiplier taking a value to e2m1 units (0 when sf is 0)
  bool finite;
};

// Scale of a block from the bit pattern of its largest magnitude.
__device__ __forceinline__ Fp4Scale fp4_block_scale(uint32_t amax_bits, float gs) {
  Fp4Scale s;
  if (amax_bits >= 0x7F800000u) {
    s.code = 0x7Fu;
    s.enc = 0.f;
    s.finite = false;
    return s;
  }
  const float t = __fdiv_rn(__uint_as_float(amax_bits) * gs, 6.0f);
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}"
      : "=h"(r)
      : "f"(0.f), "f"(t));   // t lands in the low byte
  s.code = r & 0xFFu;
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(s.code)));
  const float sf = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  s.enc = sf > 0.f ? __fdiv_rn(gs, sf) : 0.f;
  s.finite = true;
  return s;
}

// v0 (low nibble) and v1 (high nibble), already in e2m1 units, as one byte.
__device__ __forceinline__ uint32_t e2m1x2_byte(float v0, float v1) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tmov.b32 %0, {b, b, b, b};\n\t}"
      : "=r"(r)
      : "f"(v1), "f"(v0));
  return r & 0xFFu;
}

// Eight values in e2m1 units as four bytes (value 2i in the low nibble of byte i).
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// One thread holds a whole block of 16 values: returns the scale byte and
// writes the 16 codes as 8 bytes (value i in nibble i).
__device__ __forceinline__ uint32_t fp4_quantize16(const float (&v)[16], float gs, uint2& codes) {
  uint32_t a = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = max(a, abs_bits(v[i]));
  const Fp4Scale s = fp4_block_scale(a, gs);
  float t[2][8];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i >> 3][i & 7] = s.finite ? v[i] * s.enc : 0.f;
  codes.x = e2m1x8(t[0]);
  codes.y = e2m1x8(t[1]);
  return s.code;
}

// Lane-group form: each of 16 consecutive lanes (lanes 0-15 or 16-31 of a
// warp; all 32 lanes must call it together) holds one value of a block.
// Returns the scale byte (the same on the 16 lanes); `pair` receives, on even
// lanes, the byte holding this lane's code (low nibble) and the next lane's.
__device__ __forceinline__ uint32_t fp4_quantize_lane16(float v, float gs, uint32_t& pair) {
  uint32_t a = abs_bits(v);
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
  const Fp4Scale s = fp4_block_scale(a, gs);
  const float t = s.finite ? v * s.enc : 0.f;
  const float tn = __shfl_down_sync(0xffffffffu, t, 1);
  pair = e2m1x2_byte(t, tn);
  return s.code;
}

}  // namespace fn
