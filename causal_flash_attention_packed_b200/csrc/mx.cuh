// MXFP8 arithmetic shared by the quantiser and the MXFP8 attention kernels:
// E8M0 scale exponents, E4M3 conversion and the block-scaled tcgen05 MMA.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fapk.h"
#include "ptx.cuh"

namespace fapk {

// Scale exponent X of a block with maximum magnitude `amax` (a non-negative
// finite float); floor(log2 amax) is read from the bit pattern.
//  FAPK_SCALE_RCEIL: smallest X with amax * 2^-X <= 448 (one more than
//                    floor(log2 amax) - 8 when the significand exceeds 1.75).
//  FAPK_SCALE_OCP:   floor(log2 amax) - 8.
// Clamped to [-127, 127]; amax == 0 gives -127.
__device__ __forceinline__ int mx_block_exponent(float amax, int rule) {
  const uint32_t b = __float_as_uint(amax);
  if (b == 0u) return -127;
  const int E = (int)((b >> 23) & 0xFFu);
  const uint32_t M = b & 0x7FFFFFu;
  int e;
  bool above;
  if (E != 0) {
    e = E - 127;
    above = M > 0x600000u;  // 1 + M / 2^23 > 1.75
  } else {                  // subnormal: M * 2^-149
    const int n = 32 - __clz(M);
    e = n - 150;
    above = 4ull * M > (7ull << (n - 1));
  }
  int X = e - 8 + ((rule == FAPK_SCALE_RCEIL && above) ? 1 : 0);
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^-X as a float (X in [-126, 126]; exponent field stays normal).
__device__ __forceinline__ float mx_pow2_neg(int X) { return __uint_as_float((uint32_t)(127 - X) << 23); }
// 2^X as a float (X in [-126, 127]).
__device__ __forceinline__ float mx_pow2(int X) { return __uint_as_float((uint32_t)(127 + X) << 23); }

// Two E4M3 codes (round to nearest even, saturating to +-448): lo in the low byte.
__device__ __forceinline__ uint32_t mx_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Bytewise: a code whose magnitude is zero becomes 0x00 (no negative zero).
__device__ __forceinline__ uint32_t mx_canon_zero(uint32_t w) {
  const uint32_t nz = ((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & 0x80808080u;
  return (w & 0x7F7F7F7Fu) | (w & nz);
}

// Two E4M3 codes (low 16 bits of `c2`) -> two floats (exact).
__device__ __forceinline__ void mx_decode2(uint32_t c2, float& lo, float& hi) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)c2));
  const __half2 h = *reinterpret_cast<__half2*>(&h2);
  lo = __low2float(h);
  hi = __high2float(h);
}

// Eight values -> eight codes with scale exponent X.
__device__ __forceinline__ uint2 encode8(const float (&f)[8], int X) {
  const float s = mx_pow2_neg(X);
  uint32_t a = mx_e4m3x2(f[0] * s, f[1] * s) | (mx_e4m3x2(f[2] * s, f[3] * s) << 16);
  uint32_t b = mx_e4m3x2(f[4] * s, f[5] * s) | (mx_e4m3x2(f[6] * s, f[7] * s) << 16);
  return make_uint2(mx_canon_zero(a), mx_canon_zero(b));
}

// Dequantised values decode(code) * 2^X of eight codes, as bf16 (exact for
// every value within the bf16 range).
__device__ __forceinline__ uint4 dequant8_bf16(uint2 codes, int X) {
  const float sc = mx_pow2(X < -126 ? -126 : X);
  const float extra = X < -126 ? 0.5f : 1.f;  // X = -127 only for all-zero blocks
  const uint32_t w[2] = {codes.x, codes.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float a, b, c, d;
    mx_decode2(w[i] & 0xFFFFu, a, b);
    mx_decode2(w[i] >> 16, c, d);
    o[2 * i] = pack_bf16x2(a * sc * extra, b * sc * extra);
    o[2 * i + 1] = pack_bf16x2(c * sc * extra, d * sc * extra);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// max(|a|, |b|) in magnitude (the sign of the result is that of neither; take
// its absolute value at the end of a chain).
__device__ __forceinline__ float max_abs_xs(float a, float b) {
  float r;
  asm("max.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// MX quantisation of one 32-value block of a computed operand (P or dS of the
// attention kernels), held as 16 packed pairs: 8 code words and the scale
// byte.  Same codes as the quantiser except that a value that rounds to zero
// from below keeps the code 0x80 (-0), which adds nothing to an MMA.
// kNonneg: every value is >= 0, so the block maximum needs no |.|.
template <bool kNonneg>
__device__ __forceinline__ uint32_t mx_quant32_pairs(const uint64_t (&v)[16], int rule, uint32_t (&codes)[8]) {
  float x[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) f2_unpack(v[i], x[2 * i], x[2 * i + 1]);
  float amax;
  if (kNonneg) {
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = fmaxf(x[k], x[4 + k]);
#pragma unroll
    for (int c = 8; c < 32; c += 8) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float r;
        asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m[k]), "f"(x[c + k]), "f"(x[c + 4 + k]));
        m[k] = r;
      }
    }
    amax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
  } else {
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = max_abs_xs(x[k], x[4 + k]);
#pragma unroll
    for (int c = 8; c < 32; c += 4) {
#pragma unroll
      for (int k = 0; k < 4; ++k) m[k] = max_abs_xs(m[k], x[c + k]);
    }
    amax = fabsf(max_abs_xs(max_abs_xs(m[0], m[1]), max_abs_xs(m[2], m[3])));
  }
  const int X = mx_block_exponent(amax, rule);
  const float sc = mx_pow2_neg(X < -126 ? -126 : X);
  const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a, b, c, d;
    f2_unpack(f2_mul(v[2 * i], sc2), a, b);
    f2_unpack(f2_mul(v[2 * i + 1], sc2), c, d);
    codes[i] = mx_e4m3x2(a, b) | (mx_e4m3x2(c, d) << 16);
  }
  return (uint32_t)(X + 127);
}

// Instruction descriptor of kind::mxf8f6f4.block_scale with E4M3 A and B,
// E8M0 scales, fp32 accumulation: [4,6) B scale-factor id, [7,10) A format
// (0 = E4M3), [10,13) B format, bit 15 A major, bit 16 B major (1 = MN),
// [17,23) N >> 3, bit 23 scale format (1 = E8M0), [24,29) M >> 4, [29,31) A
// scale-factor id, bit 31 K = 32.
__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, bool b_mn, int a_sf_id, int b_sf_id) {
  return ((uint32_t)b_sf_id << 4) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24) | ((uint32_t)a_sf_id << 29);
}

// D[tmem] (+)= (A * SFA) (B * SFB), both operands from shared memory, scale
// factors from TMEM.  The K-block index of the scale bytes sits in the top two
// bits of the scale-factor addresses and in the descriptor's id fields.
__device__ __forceinline__ void mma_mxf8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// A scale block copied by tmem_cp_sf takes 4 TMEM columns (128 bits per lane).
// True when the blocks starting at cols[] are pairwise disjoint, start at or
// after first_free (the end of the accumulators) and end within 512 columns.
template <int N>
constexpr bool sf_cols_ok(const uint32_t (&cols)[N], uint32_t first_free) {
  for (int i = 0; i < N; ++i) {
    if (cols[i] < first_free || cols[i] + 4 > 512) return false;
    for (int j = 0; j < i; ++j)
      if (cols[i] < cols[j] + 4 && cols[j] < cols[i] + 4) return false;
  }
  return true;
}

// Copy a 512-byte scale-factor block from shared memory into 4 TMEM columns,
// replicated into all four 32-lane quarters.  The block holds the 4 scale
// bytes (one per 32-element K block) of 128 rows: row r = r0 + 32 r1 at byte
// 16 r0 + 4 r1 + k.  After the copy, column c of every lane quarter holds in
// lane r0 the word of row r0 + 32 c.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint32_t smem_block) {
  // no-swizzle K-major descriptor: 8-row core matrices of 16-byte rows,
  // 128 bytes apart
  uint64_t d = 0;
  d |= (uint64_t)((smem_block >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;           // leading offset (unused: one 16-byte column)
  d |= (uint64_t)(128 >> 4) << 32;  // stride between 8-row core matrices
  d |= (uint64_t)1 << 46;           // version
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// 4 scale bytes of token t (per-token form), or the neutral byte 127 (2^0)
// past the end of the tensor.
__device__ __forceinline__ uint32_t pt_word(const uint8_t* spt, int t, int T, int H, int h) {
  return t < T ? __ldg(reinterpret_cast<const uint32_t*>(spt + ((size_t)t * H + h) * 4)) : 0x7F7F7F7Fu;
}

// 4 scale bytes of document-local token block `blk` of document `doc`
// (token-block form); 127s past the document's last block.
__device__ __forceinline__ uint32_t tb_word(const uint8_t* stb, int s, int e, int doc, int blk, int H, int g) {
  if (32 * blk >= e - s) return 0x7F7F7F7Fu;
  const size_t slot = (size_t)(s >> 5) + doc + blk;
  return __ldg(reinterpret_cast<const uint32_t*>(stb + (slot * H + g) * 4));
}

}  // namespace fapk
