// codec.cuh -- the MXFP8 block encoding shared by the quantisers and the
// GEMM epilogue that quantises its own output.
//
// MXFP8 (opensourcebeat.com, "Enabling up to 41% faster pre-training: MXFP8
// and DeepEP ...", FAQ; OCP MX v1.0): a block of 32 elements shares the E8M0
// scale byte s + 127 with s = floor(log2 amax) - 8 clamped to [-127, 127];
// each element becomes the E4M3 code of x * 2^-s, rounded to nearest even and
// saturated to +-448.  A block holding Inf/NaN gets the NaN scale 0xFF and
// NaN codes.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace mxf8 {

// Scale byte from the largest |x| given as bf16 magnitude bits.  For a normal
// amax with biased exponent E, floor(log2 amax) = E - 127, so s = E - 135 and
// the byte is E - 8; E <= 8 (including zero and bf16 subnormals, E = 0)
// clamps to s = -127, byte 0.  E = 255 (Inf/NaN) gives the NaN scale 0xFF.
__device__ __forceinline__ uint32_t scale_byte(uint32_t amax_bits) {
  const uint32_t e = (amax_bits >> 7) & 0xFFu;
  if (e == 0xFFu) return 0xFFu;
  return e > 8u ? e - 8u : 0u;
}

// 2^-s as an fp32 for a finite scale byte b = s + 127 (exponent field
// 254 - b lies in [8, 254], so the value is a normal number and x * 2^-s is
// exact whenever it is representable).
__device__ __forceinline__ float inv_scale(uint32_t b) { return __uint_as_float((254u - b) << 23); }

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t amax_bits8(const uint4& v) {
  const uint32_t k = 0x7FFF7FFFu;
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & k, v.y & k), __vmaxu2(v.z & k, v.w & k));
  return max(m & 0xFFFFu, m >> 16);
}

// Codes of two bf16 (packed in w) scaled by f: two bytes, low element first.
__device__ __forceinline__ uint32_t enc2(uint32_t w, float f) {
  return cvt_e4m3x2(__fmul_rn(bf_lo(w), f), __fmul_rn(bf_hi(w), f));
}

__device__ __forceinline__ uint2 encode8(const uint4& v, uint32_t sb) {
  if (sb == 0xFFu) return make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
  const float f = inv_scale(sb);
  return make_uint2(enc2(v.x, f) | (enc2(v.y, f) << 16), enc2(v.z, f) | (enc2(v.w, f) << 16));
}

// Codes of a non-finite colwise block, 4 rows per word (word j: rows 4j..4j+3,
// low byte first): 0x7F for each of the block's `valid` real rows, 0x00 for
// the pad rows of a group's short last block.
__device__ __forceinline__ uint32_t nan_codes4(int j, int valid) {
  const int n = valid - 4 * j;
  if (n >= 4) return 0x7F7F7F7Fu;
  if (n <= 0) return 0u;
  return 0x7F7F7F7Fu & ((1u << (8 * n)) - 1u);
}

}  // namespace mxf8
