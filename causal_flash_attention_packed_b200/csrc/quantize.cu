// MXFP8 quantisation of a bf16 [T][H][d] tensor into E4M3 codes with E8M0
// scales (FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri":
// MXFP8 path, token-block scaling, document-local scales, fused quantisation).
//
// One CTA per (token-block slot, head, tensor).  Block m of document k
// (tokens [s_k + 32m, min(s_k + 32m + 32, e_k))) lives in slot
// floor(s_k/32) + k + m; this slot numbering is strictly increasing in k, so a
// CTA finds its document by binary search and exits if its slot holds no
// block.  The CTA reads the block's 32 tokens x d channels of one head once
// and writes both forms:
//   per-token form   -- one scale per (token, 32 channels)
//   token-block form -- one scale per (32 tokens, 32 channels)
// One launch can quantise two tensors of the same shape (K and V): blockIdx.z
// picks the job.  The backward's variant also reads O and its bf16 residual in
// the same pass and writes D_i = dO_i . (O_i + residual_i), so that dO is read
// once for D and for its quantisation.  The mixed NVFP4/FP8 path's K job also
// writes K's NVFP4 form (16-channel blocks inside one token) in the same pass.
// The kernel is bound by HBM traffic: 2 bytes read and 1 + 1/32 bytes written
// per element and form (plus 4 bytes read per element of O for D).
#include <cuda_bf16.h>

#include "internal.h"
#include "mx.cuh"
#include "nv.cuh"
#include "ptx.cuh"

namespace fapk {

namespace {

template <int D, bool kDelta>
__global__ void __launch_bounds__(128) quantize_mxfp8_kernel(const QuantJobs jobs, const int32_t* __restrict__ cu,
                                                             int n_docs, int forms, int rule, DeltaArgs da) {
  constexpr int TPR = D / 8;      // threads per token row (8 channels each)
  constexpr int RPP = 128 / TPR;  // token rows per pass
  constexpr int NP = 32 / RPP;    // passes over the 32-token block
  constexpr int NG = D / 32;      // channel groups
  const QuantJob job = blockIdx.z ? jobs.job[1] : jobs.job[0];  // no dynamic index into the parameters
  const __nv_bfloat16* __restrict__ x = job.x;
  const int H = job.H;
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
  // the forms may be laid out with a row of 128 codes and 4 scale groups per
  // (token, head) whatever D (job.padded): channels D..127 then hold zero
  // codes and their groups the scale byte 127
  const bool pad = job.padded && D < 128;
  const size_t cstride = pad ? (size_t)H * 128 : row_stride;
  const size_t ccol = pad ? (size_t)h * 128 + c8 * 8 : col;
  const int sgroups = pad ? 4 : NG;

  uint4 raw[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int row = r0 + p * RPP;
    raw[p] = row < nb ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + row) * row_stride + col))
                      : make_uint4(0, 0, 0, 0);
  }
  float f[NP][8];
#pragma unroll
  for (int p = 0; p < NP; ++p) unpack8(raw[p], f[p]);
  if (kDelta) {
    // D of each row: this thread's 8 channels, then the row's TPR threads
    // (adjacent lanes) by a butterfly
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int row = r0 + p * RPP;
      float acc = 0.f;
      if (row < nb) {
        const size_t off = (size_t)(t0 + row) * row_stride + col;
        float fo[8], fr[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(da.o + off)), fo);
        unpack8(__ldg(reinterpret_cast<const uint4*>(da.o_resid + off)), fr);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += (fo[i] + fr[i]) * f[p][i];
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
      if (c8 == 0 && row < nb) da.delta[(size_t)h * da.T + t0 + row] = acc;
    }
  }
  float amax_tb = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[p][i]));
    // the 4 threads of one 32-channel group are adjacent lanes; a lane pair
    // holds one 16-channel block
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    const int row = r0 + p * RPP;
    if (job.nvv && row < nb) {
      // NVFP4 form: both lanes of the pair derive the same scale from the
      // block maximum; each writes its 8 codes, the even lane the scale byte.
      // The row always has 128 channels: for D = 64 channels 64..127 are zero
      // codes with scale 0, which add nothing to a product.
      float r;
      const uint32_t sb = nv_block_scale(a, job.nv_six_g, job.nv_g, r);
      const size_t t = (size_t)(t0 + row);
      *reinterpret_cast<uint32_t*>(job.nvv + (t * H + h) * 64 + c8 * 4) = nv_codes8(f[p], r);
      if ((c8 & 1) == 0) job.nvs[(t * H + h) * 8 + (c8 >> 1)] = (uint8_t)sb;
      if (D < 128) {
        *reinterpret_cast<uint32_t*>(job.nvv + (t * H + h) * 64 + D / 2 + c8 * 4) = 0u;
        if ((c8 & 1) == 0) job.nvs[(t * H + h) * 8 + D / 16 + (c8 >> 1)] = 0;
      }
    }
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    if ((forms & FAPK_FORM_PT) && row < nb) {
      const int X = mx_block_exponent(a, rule);
      const size_t t = (size_t)(t0 + row);
      const uint2 codes = encode8(f[p], X);
      *reinterpret_cast<uint2*>(job.vpt + t * cstride + ccol) = codes;
      if (pad) {
        *reinterpret_cast<uint2*>(job.vpt + t * cstride + ccol + D) = make_uint2(0u, 0u);
        if ((c8 & 3) == 0) job.spt[(t * H + h) * sgroups + NG + (c8 >> 2)] = (uint8_t)127;
      }
      if (job.deq) *reinterpret_cast<uint4*>(job.deq + t * row_stride + col) = dequant8_bf16(codes, X);
      if ((c8 & 3) == 0) job.spt[(t * H + h) * sgroups + (c8 >> 2)] = (uint8_t)(X + 127);
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
    if (row < nb) {
      *reinterpret_cast<uint2*>(job.vtb + (size_t)(t0 + row) * cstride + ccol) = encode8(f[p], X);
      if (pad) *reinterpret_cast<uint2*>(job.vtb + (size_t)(t0 + row) * cstride + ccol + D) = make_uint2(0u, 0u);
    }
  }
  if (threadIdx.x < NG) {
    const int gg = threadIdx.x;
    const float ag = fmaxf(fmaxf(red[0][gg], red[1][gg]), fmaxf(red[2][gg], red[3][gg]));
    job.stb[((size_t)slot * H + h) * sgroups + gg] = (uint8_t)(mx_block_exponent(ag, rule) + 127);
    if (pad) job.stb[((size_t)slot * H + h) * sgroups + NG + gg] = (uint8_t)127;
  }
}

template <bool kDelta>
cudaError_t launch_jobs(const QuantJobs& jobs, int n_jobs, int T, int d, const int32_t* cu, int n_docs, int forms,
                        int rule, const DeltaArgs& da, cudaStream_t stream) {
  int H = 0;
  for (int i = 0; i < n_jobs; ++i) H = max(H, jobs.job[i].H);
  const dim3 grid((unsigned)(T / 32 + n_docs), (unsigned)H, (unsigned)n_jobs);
  if (d == 128)
    quantize_mxfp8_kernel<128, kDelta><<<grid, 128, 0, stream>>>(jobs, cu, n_docs, forms, rule, da);
  else
    quantize_mxfp8_kernel<64, kDelta><<<grid, 128, 0, stream>>>(jobs, cu, n_docs, forms, rule, da);
  note_launches(1);
  return cudaGetLastError();
}

// NVFP4 of a [T][H][128] tensor: one thread per (token, head, 16-channel block).
__global__ void __launch_bounds__(256) quantize_nvfp4_kernel(const __nv_bfloat16* __restrict__ x, long long n_blocks,
                                                             float six_g, float g, uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n_blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + b * 16);
  float f[16];
  unpack8(__ldg(src), *reinterpret_cast<float(*)[8]>(&f[0]));
  unpack8(__ldg(src + 1), *reinterpret_cast<float(*)[8]>(&f[8]));
  uint32_t c[2];
  scales[b] = (uint8_t)nv_quant16(f, six_g, g, c);
  *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(c[0], c[1]);
}

}  // namespace

cudaError_t launch_quantize_nvfp4(const void* x, int T, int H, float g, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream) {
  const long long n_blocks = (long long)T * H * 8;
  if (n_blocks == 0) return cudaSuccess;
  quantize_nvfp4_kernel<<<(unsigned)((n_blocks + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), n_blocks, 6.0f * g, g, codes, scales);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp8(const void* x, int T, int H, int d, const int32_t* cu, int n_docs,
                                  int forms, int rule, uint8_t* vtb, uint8_t* stb, uint8_t* vpt,
                                  uint8_t* spt, cudaStream_t stream, void* deq_pt_bf16) {
  QuantJobs jobs;
  jobs.job[0] = QuantJob{static_cast<const __nv_bfloat16*>(x), H, vtb, stb, vpt, spt,
                         static_cast<__nv_bfloat16*>(deq_pt_bf16), false};
  return launch_jobs<false>(jobs, 1, T, d, cu, n_docs, forms, rule, DeltaArgs{}, stream);
}

cudaError_t launch_quantize_jobs(const QuantJobs& jobs, int n_jobs, int T, int d, const int32_t* cu, int n_docs,
                                 int forms, int rule, cudaStream_t stream) {
  return launch_jobs<false>(jobs, n_jobs, T, d, cu, n_docs, forms, rule, DeltaArgs{}, stream);
}

cudaError_t launch_quantize_with_delta(const QuantJob& job, int T, int d, const int32_t* cu, int n_docs, int rule,
                                       const DeltaArgs& da, cudaStream_t stream) {
  QuantJobs jobs;
  jobs.job[0] = job;
  return launch_jobs<true>(jobs, 1, T, d, cu, n_docs, FAPK_FORM_TB | FAPK_FORM_PT, rule, da, stream);
}

}  // namespace fapk
