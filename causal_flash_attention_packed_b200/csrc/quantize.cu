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
#include "mx.cuh"
#include "ptx.cuh"

namespace fapk {

namespace {

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

template <int D>
__global__ void __launch_bounds__(128) quantize_mxfp8_kernel(
    const __nv_bfloat16* __restrict__ x, int H, const int32_t* __restrict__ cu, int n_docs, int forms,
    int rule, uint8_t* __restrict__ vtb, uint8_t* __restrict__ stb, uint8_t* __restrict__ vpt,
    uint8_t* __restrict__ spt, __nv_bfloat16* __restrict__ deq_pt) {
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
      const int X = mx_block_exponent(a, rule);
      const size_t t = (size_t)(t0 + row);
      const uint2 codes = encode8(f[p], X);
      *reinterpret_cast<uint2*>(vpt + t * row_stride + col) = codes;
      if (deq_pt) *reinterpret_cast<uint4*>(deq_pt + t * row_stride + col) = dequant8_bf16(codes, X);
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
  const int X = mx_block_exponent(a, rule);
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int row = r0 + p * RPP;
    if (row < nb)
      *reinterpret_cast<uint2*>(vtb + (size_t)(t0 + row) * row_stride + col) = encode8(f[p], X);
  }
  if (threadIdx.x < NG) {
    const int gg = threadIdx.x;
    const float ag = fmaxf(fmaxf(red[0][gg], red[1][gg]), fmaxf(red[2][gg], red[3][gg]));
    stb[((size_t)slot * H + h) * NG + gg] = (uint8_t)(mx_block_exponent(ag, rule) + 127);
  }
}

}  // namespace

cudaError_t launch_quantize_mxfp8(const void* x, int T, int H, int d, const int32_t* cu, int n_docs,
                                  int forms, int rule, uint8_t* vtb, uint8_t* stb, uint8_t* vpt,
                                  uint8_t* spt, cudaStream_t stream, void* deq_pt_bf16) {
  const dim3 grid((unsigned)(T / 32 + n_docs), (unsigned)H);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* dq = static_cast<__nv_bfloat16*>(deq_pt_bf16);
  if (d == 128)
    quantize_mxfp8_kernel<128><<<grid, 128, 0, stream>>>(xb, H, cu, n_docs, forms, rule, vtb, stb, vpt, spt, dq);
  else
    quantize_mxfp8_kernel<64><<<grid, 128, 0, stream>>>(xb, H, cu, n_docs, forms, rule, vtb, stb, vpt, spt, dq);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
