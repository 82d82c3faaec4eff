// Fused QKV projection with MXFP8 quantisation in its epilogue, for sm_100a.
//
// [Q | K | V] = X W^T in one GEMM over the packed tokens ("GPT Kernel
// Programlama: MatMul, Softmax ve Attention Hesabi", sec. 2: the three
// projections run as one fused QKV projection, so X is read once and fewer
// kernels are launched), with the quantisation of K and V done by the GEMM's
// epilogue (FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri":
// fused quantisation, document-local scales over packed layouts): the
// attention forward then reads K and V in both MX forms without a
// quantisation pass of its own.
//
//   x [T][Dm] bf16, w [N][Dm] bf16 with N = (Hq + 2 Hkv) d (rows of W: the Q
//   heads, then the K heads, then the V heads), d = 128.
//   q [T][Hq][d], k, v [T][Hkv][d] bf16 (the fp32 products rounded to
//   nearest even); K and V also in token-block and per-token MX form,
//   quantised from those bf16 values, in the layout of fapk_quantize_mxfp8.
//
// Design (persistent, 1 CTA per SM, 192 threads):
//  * work unit = (document, 128-row tile, pair of heads of Q, K or V; 256
//    output columns): the row tiles
//    start at the document start (the scheduler's per-document tiles), so
//    each document-local 32-token block lies inside one tile and the
//    epilogue forms its token-block scale from its own rows; rows past the
//    document end belong to the next document and are not stored;
//  * warp 0: TMA loads of the X tile and the 256 W rows (64 channels of Dm
//    per stage, 128-byte swizzle) into a ring of kStages stages;
//  * warp 1, one lane: tcgen05 MMAs (128 x 256 x 16, bf16, fp32 accumulation
//    in TMEM), two accumulator buffers of 256 columns so that the epilogue of
//    one unit overlaps the MMAs of the next.  A 128 x 256 MMA reads 12 KB of
//    operands in 128 cycles and the stage's copies write as much again: 192
//    bytes per cycle of shared memory against the 128 it has, a ceiling of
//    about two thirds of the MMA rate (half with 128-column tiles);
//  * warps 2-5: epilogue, one thread per output row (TMEM lane): fp32 -> bf16,
//    and for K and V heads the per-token form (per 32 channels) and the
//    token-block form (the warp's 32 rows are one token block) of each
//    32-channel group; for the mixed NVFP4/FP8 path K's NVFP4 form (two
//    16-channel blocks per group) instead of its MX forms.
#include <cuda_bf16.h>

#include "internal.h"
#include "mx.cuh"
#include "nv.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace fapk {

namespace {

constexpr int kThreads = 192;
constexpr int kLoadWarp = 0, kMmaWarp = 1;  // warps 2-5: epilogue
constexpr int kStages = 4;
constexpr int kBoxBytes = 128 * 64 * 2;     // 128 rows x 64 bf16
constexpr int kStageBytes = 3 * kBoxBytes;  // X tile and two W boxes (256 rows)
// bars: full[S], empty[S], acc_full[2], acc_empty[2], fin; the unit ring's full[8], empty[8]
constexpr int kNumBars = 2 * kStages + 5 + 2 * kUnitRing;
constexpr int kSmemBytes = kStages * kStageBytes + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory exceeds the 227 KB a CTA may use");

struct Params {
  const int32_t* cu;
  SchedView sched;
  __nv_bfloat16 *q, *k, *v;
  uint8_t *k_vtb, *k_stb, *k_vpt, *k_spt;
  uint8_t *v_vtb, *v_stb, *v_vpt, *v_spt;
  uint8_t *k_nvv, *k_nvs;  // mixed path: K's NVFP4 form instead of its MX forms (null: MX)
  float nv_g_k, nv_six_g_k;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int T, Dm, Hq, Hkv, n_heads;  // n_heads = Hq + 2 Hkv: the unit's head index runs over Q, K, V heads
  int rule;
};

__global__ void __launch_bounds__(kThreads, 1)
    qkv_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* fin = acc_full + 4;
  const UnitRing ring{reinterpret_cast<int*>(bars + kNumBars) + 4, bars + kNumBars - 2 * kUnitRing,
                      bars + kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);  // the epilogue warps
    }
    mbar_init(fin, 1);
    unit_ring_init(ring, 1 + 4);  // the MMA thread and the epilogue warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{p.status, abort_flag, p.timeout_ns};
  const UnitSpace us = unit_space(p.sched, (p.n_heads + 1) / 2, kSchedKV);  // head pairs
  const int n_units = us.n_units();
  const int n_k = (p.Dm + 63) / 64;  // 64-channel steps along Dm (the last one zero-filled past Dm)

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk) {
        const UnitInfo un = unit_produce(ring, us, p.cu, p.sched.next, uk, wd);
        if (un.w < 0 || un.w >= n_units) break;
        const int t0 = un.s + 128 * un.tile, n0 = 256 * un.h;
        for (int kc = 0; kc < n_k; ++kc, ++it) {
          const int st = it % kStages;
          const uint32_t use = it / kStages;
          if (use > 0 && !mbar_wait(empty + st, (use - 1) & 1, wd, 1)) { ok = false; break; }
          uint8_t* sb = smem + st * kStageBytes;
          mbar_arrive_expect_tx(full + st, kStageBytes);
          tma_load_3d(sb, &tm_x, full + st, 64 * kc, 0, t0);
          // W rows n0 .. n0 + 255 (past the last head: zero-filled)
          tma_load_3d(sb + kBoxBytes, &tm_w, full + st, 64 * kc, 0, n0);
          tma_load_3d(sb + 2 * kBoxBytes, &tm_w, full + st, 64 * kc, 0, n0 + 128);
        }
      }
      for (uint32_t i = (it > kStages ? it - kStages : 0); i < it; ++i)
        drain_wait(full + (i % kStages), (i / kStages) & 1, p.timeout_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
      uint32_t it = 0, unit_i = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        if (un.w < 0 || un.w >= n_units) break;
        const int buf = unit_i & 1;
        const uint32_t bu = unit_i >> 1;  // uses of this accumulator buffer so far
        if (bu > 0 && !mbar_wait(acc_empty + buf, (bu - 1) & 1, wd, 2)) break;
        tc_fence_after();
        const uint32_t acc = tmem + 256 * buf;
        for (int kc = 0; kc < n_k; ++kc, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(full + st, (it / kStages) & 1, wd, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * kStageBytes);
          const uint64_t da = sdesc_sw128(sa, 16, 1024), db = sdesc_sw128(sa + kBoxBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(acc, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          tc_commit(empty + st);
        }
        if (!ok) break;
        tc_commit(acc_full + buf);
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    const int row = quarter * 32 + lane;
    uint32_t unit_i = 0;
    for (uint32_t uk = 0;; ++uk, ++unit_i) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      if (un.w < 0 || un.w >= n_units) break;
      const int buf = unit_i & 1;
      if (!warp_wait(acc_full + buf, (unit_i >> 1) & 1, wd, 4)) break;
      tc_fence_after();
      const int t = un.s + 128 * un.tile + row;
      const bool valid = t < un.e;
      for (int half = 0; half < 2; ++half) {
        // the head of these 128 columns: Q heads, then K heads, then V heads
        const int hh = 2 * un.h + half;
        if (hh >= p.n_heads) break;  // an odd head count leaves the last pair half empty
        const bool is_q = hh < p.Hq, is_k = !is_q && hh < p.Hq + p.Hkv;
        const int head = is_q ? hh : (is_k ? hh - p.Hq : hh - p.Hq - p.Hkv);
        const int H = is_q ? p.Hq : p.Hkv;
        __nv_bfloat16* out = is_q ? p.q : (is_k ? p.k : p.v);
        uint8_t* vtb = is_k ? p.k_vtb : p.v_vtb;
        uint8_t* stb = is_k ? p.k_stb : p.v_stb;
        uint8_t* vpt = is_k ? p.k_vpt : p.v_vpt;
        uint8_t* spt = is_k ? p.k_spt : p.v_spt;
        const size_t orow = ((size_t)t * H + head) * 128;
        const uint32_t lane_addr = tmem + 256 * buf + 128 * half + ((uint32_t)(quarter * 32) << 16);
        for (int g = 0; g < 4; ++g) {
          // 32 channels of this row: fp32 -> bf16 (round to nearest even)
          uint32_t r[32];
          tmem_ld32(lane_addr + 32 * g, r);
          tmem_wait_ld(r);
          uint32_t b[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) b[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(out + orow + 32 * g);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(b[4 * e], b[4 * e + 1], b[4 * e + 2], b[4 * e + 3]);
          }
          if (is_q) continue;
          if (is_k && p.k_nvv) {
            // NVFP4 form of K (two 16-channel blocks), quantised as fapk_quantize_nvfp4 does
            if (valid) {
              float f[4][8];
#pragma unroll
              for (int c = 0; c < 4; ++c) unpack8(make_uint4(b[4 * c], b[4 * c + 1], b[4 * c + 2], b[4 * c + 3]), f[c]);
              uint32_t c0[2], c1[2];
              const uint32_t s0 = nv_quant16(&f[0][0], p.nv_six_g_k, p.nv_g_k, c0);
              const uint32_t s1 = nv_quant16(&f[2][0], p.nv_six_g_k, p.nv_g_k, c1);
              const size_t nrow = (size_t)t * H + head;
              *reinterpret_cast<uint4*>(p.k_nvv + nrow * 64 + 16 * g) = make_uint4(c0[0], c0[1], c1[0], c1[1]);
              *reinterpret_cast<uint16_t*>(p.k_nvs + nrow * 8 + 2 * g) = (uint16_t)(s0 | (s1 << 8));
            }
            continue;
          }
          // the bf16 values as floats, quantised exactly as fapk_quantize_mxfp8 does
          float f[4][8];
          float a = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            unpack8(make_uint4(b[4 * c], b[4 * c + 1], b[4 * c + 2], b[4 * c + 3]), f[c]);
#pragma unroll
            for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[c][i]));
          }
          if (!valid) a = 0.f;  // rows of the next document take no part in this block's scale
          // per-token form
          const int X = mx_block_exponent(a, p.rule);
          if (valid) {
            uint2 cw[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) cw[c] = encode8(f[c], X);
            uint4* dst = reinterpret_cast<uint4*>(vpt + orow + 32 * g);
            dst[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
            dst[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
            spt[((size_t)t * H + head) * 4 + g] = (uint8_t)(X + 127);
          }
          // token-block form: the warp's 32 rows are one document-local block
          float atb = a;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) atb = fmaxf(atb, __shfl_xor_sync(0xFFFFFFFFu, atb, off));
          const int Xtb = mx_block_exponent(atb, p.rule);
          if (valid) {
            uint2 cw[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) cw[c] = encode8(f[c], Xtb);
            uint4* dst = reinterpret_cast<uint4*>(vtb + orow + 32 * g);
            dst[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
            dst[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
          }
          const int t_blk = un.s + 128 * un.tile + 32 * quarter;  // first token of the warp's block
          if (lane == 0 && t_blk < un.e) {
            const size_t slot = (size_t)(un.s >> 5) + un.doc + 4 * un.tile + quarter;
            stb[(slot * H + head) * 4 + g] = (uint8_t)(Xtb + 127);
          }
        }
      }
      tc_fence_before();
      warp_arrive(acc_empty + buf);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_qkv_proj(const QkvProjArgs& a, cudaStream_t stream) {
  const int N = (a.Hq + 2 * a.Hkv) * 128;
  CUtensorMap tx, tw;
  if (!make_tmap_thd(&tx, a.x, a.T, 1, a.Dm) || !make_tmap_thd(&tw, a.w, N, 1, a.Dm)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  Params p;
  p.cu = a.cu;
  p.sched = sched_view(a.sched);
  p.q = static_cast<__nv_bfloat16*>(a.q);
  p.k = static_cast<__nv_bfloat16*>(a.k);
  p.v = static_cast<__nv_bfloat16*>(a.v);
  p.k_vtb = a.k_vtb; p.k_stb = a.k_stb; p.k_vpt = a.k_vpt; p.k_spt = a.k_spt;
  p.v_vtb = a.v_vtb; p.v_stb = a.v_stb; p.v_vpt = a.v_vpt; p.v_spt = a.v_spt;
  p.k_nvv = a.k_nvv; p.k_nvs = a.k_nvs;
  p.nv_g_k = a.nv_g_k;
  p.nv_six_g_k = 6.0f * a.nv_g_k;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.T = a.T;
  p.Dm = a.Dm;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.n_heads = a.Hq + 2 * a.Hkv;
  p.rule = a.rule;
  const long long max_units = (long long)a.sched.max_items * ((p.n_heads + 1) / 2);
  const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
  qkv_proj_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tx, tw, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
