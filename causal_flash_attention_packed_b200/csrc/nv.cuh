// NVFP4 arithmetic of the mixed NVFP4/FP8 path (FLAMIA page, sec. "FLAMIA
// Mimarisi ve Temel Tasarim Ilkeleri": mixed NVFP4/FP8 training paths).
//
// NVFP4 (NVIDIA's format; the pages only name it): E2M1 element codes, one
// unsigned E4M3 scale per 16 consecutive channels of one token, and an fp32
// decode scale g per tensor: x ~ code * scale * g.  A block with largest
// magnitude a is quantised in fp32, every step rounded to nearest even:
//   s = E4M3(a / (6 g))        (saturating at 448; 0 for an all-zero block)
//   r = 1 / (decode(s) g)      (0 when that product is 0)
//   code_i = E2M1(x_i r)       (saturating at +-6; a zero result is code 0)
// Codes are packed two per byte, channel 2i in the low nibble of byte i.
//
// The scores of the mixed path read these operands with the block-scaled MMA
// kind::mxf4nvf4 (scale_vec::4X): K = 64 FP4 values per instruction, the 4
// scale bytes of a row's 4 blocks in one 32-bit TMEM word.
#pragma once

#include <stdint.h>

#include "mx.cuh"
#include "ptx.cuh"

namespace fapk {

// Eight E2M1 codes of x[0..8) (round to nearest even, saturating), packed
// into one word: x[2i] in the low nibble of byte i.
__device__ __forceinline__ uint32_t nv_e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5,
                                              float x6, float x7) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(w)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  // a code whose magnitude is zero becomes 0 (no negative zero)
  const uint32_t m = w & 0x77777777u;
  return m | (w & ((m + 0x77777777u) & 0x88888888u));
}

// Scale byte s of a block with largest magnitude a, and the factor r that
// takes its values to E2M1 units.  six_g = fp32(6 g).
__device__ __forceinline__ uint32_t nv_block_scale(float a, float six_g, float g, float& r) {
  const uint32_t sbyte = mx_e4m3x2(__fdiv_rn(a, six_g), 0.f) & 0xFFu;
  float dec, unused;
  mx_decode2(sbyte, dec, unused);
  const float sg = __fmul_rn(dec, g);
  r = sg > 0.f ? __frcp_rn(sg) : 0.f;
  return sbyte;
}

// Eight values of a block whose factor is r -> one word of 8 codes.
__device__ __forceinline__ uint32_t nv_codes8(const float* y, float r) {
  return nv_e2m1x8(__fmul_rn(y[0], r), __fmul_rn(y[1], r), __fmul_rn(y[2], r), __fmul_rn(y[3], r),
                   __fmul_rn(y[4], r), __fmul_rn(y[5], r), __fmul_rn(y[6], r), __fmul_rn(y[7], r));
}

// One NVFP4 block of 16 values: codes[0..1] (8 nibbles each), returns the
// E4M3 scale byte.
__device__ __forceinline__ uint32_t nv_quant16(const float* x, float six_g, float g, uint32_t (&codes)[2]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  float r;
  const uint32_t sbyte = nv_block_scale(a, six_g, g, r);
  codes[0] = nv_codes8(x, r);
  codes[1] = nv_codes8(x + 8, r);
  return sbyte;
}

// Instruction descriptor of kind::mxf4nvf4.block_scale with E2M1 A and B
// (format 1 in both fields), UE4M3 scales (bit 23 clear), both operands
// K-major, fp32 accumulation, scale-factor ids 0 (scale_vec::4X).
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= (A * SFA) (B * SFB) over K = 64 packed E2M1 values per row,
// both operands from shared memory, the 4 scale bytes per row in TMEM.
__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a 64-byte-swizzled K-major operand tile
// (rows of 64 bytes = 128 E2M1 values; 8-row groups 512 bytes apart): layout
// type 4 in bits [61,64).
__device__ __forceinline__ uint64_t sdesc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading offset (unused: one swizzle atom along K)
  d |= (uint64_t)(512 >> 4) << 32;    // stride between 8-row groups
  d |= (uint64_t)1 << 46;             // version
  d |= (uint64_t)4 << 61;
  return d;
}

// Byte offset of 16-byte chunk c (0..3) of row r in a 64-byte-swizzled tile
// of 64-byte rows (the pattern TMA's 64-byte swizzle writes).
__device__ __forceinline__ int sw64_chunk(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// The two 4-byte scale words (channels 0..63 and 64..127) of token t, head h
// of an NVFP4 scale tensor [T][H][8]; zeros past the end of the tensor.
__device__ __forceinline__ uint2 nv_scale_words(const uint8_t* s, int t, int T, int H, int h) {
  return t < T ? __ldg(reinterpret_cast<const uint2*>(s + ((size_t)t * H + h) * 8)) : make_uint2(0u, 0u);
}

}  // namespace fapk
