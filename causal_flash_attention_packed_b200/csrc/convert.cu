// bf16 -> fp16 conversion of whole tensors (HBM-bound elementwise pass).
//
// The bf16 path multiplies the probabilities P and the score gradients dS,
// which it computes in fp32, by V, dO, Q and K on the tensor cores.  bf16
// operands would round P and dS to 8 significant bits; fp16 keeps 11 at the
// same tensor-core rate, and every bf16 input of magnitude below 65504
// converts to fp16 without loss (tiny values below 2^-14 keep fewer bits,
// which moves a product by less than 2^-24 of the other factor).  Inputs at
// or above 65504 are reported (kStatusRange) rather than silently clamped.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fapk {

namespace {

// 8 bf16 -> 8 fp16; returns false if any magnitude reaches the fp16 limit.
__device__ __forceinline__ bool cvt8(const uint4& in, uint4& out) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[4];
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
    ok &= fabsf(lo) < kF16Max && fabsf(hi) < kF16Max;
    o[i] = pack_f16x2(lo, hi);
  }
  out = make_uint4(o[0], o[1], o[2], o[3]);
  return ok;
}

__global__ void __launch_bounds__(256) convert_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          long long n8, DeviceStatus* status) {
  bool ok = true;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    uint4 o;
    ok &= cvt8(__ldg(src + i), o);
    dst[i] = o;
  }
  if (!__all_sync(0xFFFFFFFFu, ok) && (threadIdx.x & 31) == 0) record_error(status, kStatusRange, 40);
}

}  // namespace

cudaError_t launch_convert_f16(const void* src, void* dst, long long n, DeviceStatus* status, int num_sms,
                               cudaStream_t stream) {
  const long long n8 = n / 8;  // every tensor here holds a multiple of 8 elements (d = 64 or 128)
  long long blocks = (n8 + 255) / 256;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  convert_f16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                          n8, status);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
