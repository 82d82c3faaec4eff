// MXFP8 quantisation of a bf16 [T][H][d] tensor into E4M3 codes with E8M0
// scales (FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri":
// MXFP8 path, token-block scaling, document-local scales).
//
// One CTA per (token-block slot, head).  Block m of document k (tokens
// [s_k + 32m, min(s_k + 32m + 32, e_k))) lives in slot floor(s_k/32) + k + m;
// this slot numbering is strictly increasing in k, so a CTA finds its
// document by binary search and exits if its slot holds no block.  The CTA
// reads the block's 32 tokens x d channels of one head once and writes both
// forms:
//   per-token form   -- one scale per (token, 32 channels)
//   token-block form -- one scale per (32 tokens, 32 channels)
// The kernel is bound by HBM traffic: 2 bytes read and 1 + 1/32 bytes written
// per element and form.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fapk {

namespace {

// Scale exponent X of a block with maximum magnitude `amax` (a non-negative
// finite float).  floor(log2 amax) is read from the bit pattern.
//  rule 0 (RCEIL): smallest X with amax * 2^-X <= 448, i.e. one more than
//                  floor(log2 amax) - 8 when the significand exceeds 1.75.
//  rule 1 (OCP):   floor(log2 amax) - 8.
// Clamped to [-127, 127]; amax == 0 gives -127.
__device__ __forceinline__ int block_exponent(float amax, int rule) {
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

// 2^-X as a float (X in [-127, 126], so the exponent field stays normal).
__device__ __forceinline__ float pow2_neg(int X) { return __uint_as_float((uint32_t)(127 - X) << 23); }

// Two E4M3 codes (round to nearest even, saturating to +-448) in the low and
// high byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// A code whose magnitude is zero becomes 0x00 (no negative zero), bytewise.
__device__ __forceinline__ uint32_t canon_zero(uint32_t w) {
  const uint32_t nz = ((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & 0x80808080u;  // bit 7: low 7 bits != 0
  return (w & 0x7F7F7F7Fu) | (w & nz);
}

// Eight values -> eight codes with scale exponent X.
__device__ __forceinline__ uint2 encode8(const float (&f)[8], int X) {
  const float s = pow2_neg(X);
  uint32_t a = e4m3x2(f[0] * s, f[1] * s) | (e4m3x2(f[2] * s, f[3] * s) << 16);
  uint32_t b = e4m3x2(f[4] * s, f[5] * s) | (e4m3x2(f[6] * s, f[7] * s) << 16);
  return make_uint2(canon_zero(a), canon_zero(b));
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(128) quantize_mxfp8_kernel(
    const __nv_bfloat16* __restrict__ x, int H, const int32_t* __restrict__ cu, int n_docs, int forms,
    int rule, uint8_t* __restrict__ vtb, uint8_t* __restrict__ stb, uint8_t* __restrict__ vpt,
    uint8_t* __restrict__ spt) {
  constexpr int TPR = D / 8;      // threads per token row (8 channels each)
  constexpr int RPP = 128 / TPR;  // token rows per pass
  constexpr int NP = 32 / RPP;    // passes over the 32-token block
  constexpr int NG = D / 32;      // channel groups
  const int slot = blockIdx.x, h = blockIdx.y;

  // document of this slot: the largest k with floor(cu[k]/32) + k <= slot
  int lo = 0, hi = n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((cu[mid] >> 5) + mid <= slot) lo = mid; else hi = mid - 1;
  }
  const int s = cu[lo], L = cu[lo + 1] - s;
  const int m = slot - ((s >> 5) + lo);
  if (m < 0 || 32 * m >= L) return;  // slot holds no block
  const int t0 = s + 32 * m, nb = min(32, L - 32 * m);

  const int c8 = threadIdx.x % TPR, r0 = threadIdx.x / TPR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t row_stride = (size_t)H * D;
  const size_t col = (size_t)h * D + c8 * 8;

  uint4 raw[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int row = r0 + p * RPP;
    raw[p] = row < nb ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + row) * row_stride + col))
                      : make_uint4(0, 0, 0, 0);
  }
  float f[NP][8];
  float amax_tb = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    unpack8(raw[p], f[p]);
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[p][i]));
    // the 4 threads of one 32-channel group are adjacent lanes
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    const int row = r0 + p * RPP;
    if ((forms & FAPK_FORM_PT) && row < nb) {
      const int X = block_exponent(a, rule);
      const size_t t = (size_t)(t0 + row);
      *reinterpret_cast<uint2*>(vpt + t * row_stride + col) = encode8(f[p], X);
      if ((c8 & 3) == 0) spt[(t * H + h) * NG + (c8 >> 2)] = (uint8_t)(X + 127);
    }
    amax_tb = fmaxf(amax_tb, a);
  }
  if (!(forms & FAPK_FORM_TB)) return;

  // token-block maximum: reduce over the rows held by this warp, then over warps
#pragma unroll
  for (int off = TPR; off < 32; off <<= 1) amax_tb = fmaxf(amax_tb, __shfl_xor_sync(0xFFFFFFFFu, amax_tb, off));
  __shared__ float red[4][NG];
  if (lane < TPR && (lane & 3) == 0) red[warp][lane >> 2] = amax_tb;
  __syncthreads();
  const int g = c8 >> 2;
  const float a = fmaxf(fmaxf(red[0][g], red[1][g]), fmaxf(red[2][g], red[3][g]));
  const int X = block_exponent(a, rule);
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int row = r0 + p * RPP;
    if (row < nb)
      *reinterpret_cast<uint2*>(vtb + (size_t)(t0 + row) * row_stride + col) = encode8(f[p], X);
  }
  if (threadIdx.x < NG) {
    const int gg = threadIdx.x;
    const float ag = fmaxf(fmaxf(red[0][gg], red[1][gg]), fmaxf(red[2][gg], red[3][gg]));
    stb[((size_t)slot * H + h) * NG + gg] = (uint8_t)(block_exponent(ag, rule) + 127);
  }
}

}  // namespace

cudaError_t launch_quantize_mxfp8(const void* x, int T, int H, int d, const int32_t* cu, int n_docs,
                                  int forms, int rule, uint8_t* vtb, uint8_t* stb, uint8_t* vpt,
                                  uint8_t* spt, cudaStream_t stream) {
  const dim3 grid((unsigned)(T / 32 + n_docs), (unsigned)H);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  if (d == 128)
    quantize_mxfp8_kernel<128><<<grid, 128, 0, stream>>>(xb, H, cu, n_docs, forms, rule, vtb, stb, vpt, spt);
  else
    quantize_mxfp8_kernel<64><<<grid, 128, 0, stream>>>(xb, H, cu, n_docs, forms, rule, vtb, stb, vpt, spt);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
