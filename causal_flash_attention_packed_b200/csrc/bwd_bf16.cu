// Backward of causal packed-document attention, bf16 operands, for sm_100a.
//
// The analytic derivative of the forward (the pages give none):
//   D_i   = dO_i . O_i
//   P_ij  = exp(S_ij - LSE_i)           (recomputed from the saved LSE)
//   dP_ij = dO_i . V_j,   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij Q_i,  dQ_i = scale sum_j dS_ij K_j
// over visible pairs only (j <= i, same document).
//
// Three kernels, all deterministic (no atomics, fixed summation order):
//  1. delta_kernel: D and -LSE log2(e) for every (token, head).
//  2. dkdv kernel: one work item per (document, 128-key tile, KV head).  For
//     each query head of the group and each query tile at or after the key
//     tile: S^T = K Q^T and dP^T = V dO^T into TMEM (one thread per key row),
//     P^T and dS^T written back into TMEM as fp16, then dV += P^T dO and
//     dK += dS^T Q with A read from TMEM.  dK, dV accumulate in TMEM across
//     the whole item (query heads of the group included) and are written once.
//  3. dq kernel: one work item per (document, 128-query tile, query head).
//     For each key tile at or before it: S = Q K^T, dP = dO V^T, dS in TMEM,
//     dQ += dS K.
// Warp roles in both gradient kernels: warp 16 loads (TMA), warp 17 issues
// tcgen05 MMAs, warps 0-15 compute P and dS (warpgroup wg on 32 columns of
// each 128x128 tile, every thread owning one TMEM lane).  Scores are read out
// of TMEM into registers and their columns released at once, so the MMAs of
// the next tile overlap the exponentials of the current one.
// Every MMA of the backward runs on fp16 operands: the prepass copies Q, K, dO
// to fp16 (V comes from the forward's ctx), which is lossless for bf16 values
// below 65504, and P and dS are packed to fp16 (11 significant bits, where
// bf16 keeps 8).  |dS| reaching 65504 is reported as kStatusRange.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "sched.cuh"

namespace fapk {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Geo {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 64 * 2;
  static constexpr int kNumBox = D / 64;
};

// ---------------------------------------------------------------------------
// 1. D = rowsum(dO * O), fp32 [Hq][T]
// ---------------------------------------------------------------------------
// O is taken as o + o_resid, the forward's bf16 output plus its rounding
// residual (about 16 significant bits).
// The same pass writes the fp16 copies of dO and Q used by the gradient MMAs
// and -LSE log2(e), the exponent offset of P in base 2.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const __nv_bfloat16* __restrict__ o_resid,
                                                    const __nv_bfloat16* __restrict__ dout,
                                                    const __nv_bfloat16* __restrict__ q,
                                                    uint4* __restrict__ do16, uint4* __restrict__ q16,
                                                    const float* __restrict__ lse, float* __restrict__ delta,
                                                    float* __restrict__ nl2, int T, int Hq,
                                                    DeviceStatus* status) {
  constexpr int TPR = D / 8;  // threads per (token, head) row
  const long long row = (long long)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int c8 = threadIdx.x % TPR;
  float acc = 0.f;
  bool in_range = true;
  if (row < (long long)T * Hq) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + c8);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + c8);
    const uint4 qq = __ldg(reinterpret_cast<const uint4*>(q + row * D) + c8);
    {
      const uint32_t wb[4] = {b.x, b.y, b.z, b.w}, wq[4] = {qq.x, qq.y, qq.z, qq.w};
      uint32_t hb[4], hq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float b0 = __uint_as_float(wb[i] << 16), b1 = __uint_as_float(wb[i] & 0xFFFF0000u);
        const float q0 = __uint_as_float(wq[i] << 16), q1 = __uint_as_float(wq[i] & 0xFFFF0000u);
        in_range &= fmaxf(fmaxf(fabsf(b0), fabsf(b1)), fmaxf(fabsf(q0), fabsf(q1))) < kF16Max;
        hb[i] = pack_f16x2(b0, b1);
        hq[i] = pack_f16x2(q0, q1);
      }
      do16[row * (D / 8) + c8] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
      q16[row * (D / 8) + c8] = make_uint4(hq[0], hq[1], hq[2], hq[3]);
    }
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(o_resid + row * D) + c8);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w}, wr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc += (__uint_as_float(wa[i] << 16) + __uint_as_float(wr[i] << 16)) * __uint_as_float(wb[i] << 16);
      acc += (__uint_as_float(wa[i] & 0xFFFF0000u) + __uint_as_float(wr[i] & 0xFFFF0000u)) *
             __uint_as_float(wb[i] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (row < (long long)T * Hq && c8 == 0) {
    const long long t = row / Hq, h = row % Hq;
    delta[h * T + t] = acc;
    nl2[h * T + t] = -(lse[h * T + t] * kLog2e);
  }
  if (!__all_sync(0xFFFFFFFFu, in_range) && (threadIdx.x & 31) == 0) record_error(status, kStatusRange, 41);
}

struct BwdParams {
  const int32_t* cu;
  SchedView sched;
  const float* lse;
  const float* delta;
  const float* nl2;  // -LSE log2(e), [Hq][T]
  void* out0;  // dkdv: dk;  dq: dq
  void* out1;  // dkdv: dv
  DeviceStatus* status;
  uint64_t timeout_ns;
  int T, Hq, Hkv;
  float scale;       // softmax scale (dK, dQ factor)
  float scale_log2;  // scale * log2(e)
  int grad_bf16;
  int wide;  // every gradient output 32-byte aligned: 32-byte stores
  unsigned long long* cta_times;  // per-CTA (start, end) records, or null
};

// ---------------------------------------------------------------------------
// 2. dK, dV
// ---------------------------------------------------------------------------
// TMEM holds dV, dK, one 128-column region that S^T and dP^T of a query tile
// use in turn, and one region for the tile's P^T and dS^T (fp16).  The compute
// warps read S^T (then dP^T) out into registers and release the region at
// once, so the MMAs run in the order S(t), dP(t), dV(t), S(t+1), dK(t),
// dP(t+1), ... and the tensor pipe has the next independent MMA group queued
// while the exponentials of a tile are computed.  Two threads issue the MMAs:
// warp 17 the scores S^T and dP^T, warp 18 the gradients dV and dK, so that a
// wait of one never leaves the tensor pipe without the other's queued work.
// 16 compute warps: warpgroup wg owns query columns [32 wg, 32 wg + 32) of
// every tile.
constexpr int kKvThreads = 608;
constexpr int kKvLoadWarp = 16;
constexpr int kKvMmaWarp = 17;   // S^T, dP^T; owns the TMEM allocation
constexpr int kKvGradWarp = 18;  // dV, dK
constexpr int kKvComputeWarps = 16;

template <int D>
struct KvCfg : Geo<D> {
  // Q and dO stream through separate rings: dO (with the tile's -LSE log2(e)
  // and D) is free once dV and dS are done, Q only after dK, so Q gets one
  // stage more
  static constexpr int kQStages = 3, kOStages = 2;
  static constexpr int kOStageBytes = Geo<D>::kTileBytes + 1024;  // dO, nl2[128], D[128]
  static constexpr int kNl2Off = Geo<D>::kTileBytes, kDeltaOff = kNl2Off + 512;
  static constexpr int kSmemTiles = (2 + kQStages) * Geo<D>::kTileBytes + kOStages * kOStageBytes;
  // TMEM: dV [0,D), dK [128,128+D), S^T / dP^T [256,384), P^T [384,448), dS^T [448,512)
  static constexpr uint32_t kDV = 0, kDK = 128, kSD = 256, kP = 384, kDS = 448;
  // bars: kv_full, kv_empty, q_full[Q], q_empty[Q], o_full[O], o_empty[O], s_full, s_free, p_ready,
  //       ds_ready, dv_done, dk_done, acc_full, acc_free, fin
  // + the unit ring's full[8] and empty[8]
  static constexpr int kNumBars = 2 + 2 * kQStages + 2 * kOStages + 9 + 2 * kUnitRing;
  // no alignment slack: the kernel checks that dynamic shared memory starts
  // on a 1024-byte boundary
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + kUnitRingBytes;
};
static_assert(KvCfg<128>::kSmemBytes <= 227 * 1024 && KvCfg<64>::kSmemBytes <= 227 * 1024,
              "shared memory of the dK/dV kernel exceeds the 227 KB a CTA may use");

struct KvItem {
  int s, e, v, g, k0, nq;  // k0: first key of the tile; query tiles v..nq-1
};

__device__ __forceinline__ KvItem kv_decode(const UnitInfo& un) {
  KvItem it;
  it.v = un.tile;
  it.g = un.h;
  it.s = un.s;
  it.e = un.e;
  it.k0 = it.s + 128 * it.v;
  it.nq = (it.e - it.s + 127) / 128;
  return it;
}

// 32 values of one TMEM row -> registers.
__device__ __forceinline__ void ld_row32(uint32_t taddr, float (&x)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld(r);
#pragma unroll
  for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(r[c]);
}

template <int D>
__global__ void __launch_bounds__(kKvThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if ((smem_u32(smem) & 1023u) != 0) {  // 128-byte swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_error(p.status, kStatusInternal, 20);
    return;
  }
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTileBytes;
  uint8_t* sQr = smem + 2 * C::kTileBytes;             // Q ring
  uint8_t* sOr = sQr + C::kQStages * C::kTileBytes;    // dO ring: dO tile, nl2[128], D[128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;
  uint64_t* q_empty = q_full + C::kQStages;
  uint64_t* o_full = q_empty + C::kQStages;
  uint64_t* o_empty = o_full + C::kOStages;
  uint64_t* s_full = o_empty + C::kOStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_ready = s_full + 2;
  uint64_t* ds_ready = s_full + 3;
  uint64_t* dv_done = s_full + 4;
  uint64_t* dk_done = s_full + 5;
  uint64_t* acc_full = s_full + 6;
  uint64_t* acc_free = s_full + 7;
  uint64_t* fin = s_full + 8;
  const UnitRing ring{reinterpret_cast<int*>(bars + C::kNumBars) + 4, bars + C::kNumBars - 2 * kUnitRing,
                      bars + C::kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < C::kQStages; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
    }
    for (int i = 0; i < C::kOStages; ++i) {
      mbar_init(o_full + i, 33);                   // lane 0's expect_tx arrive + 32 lanes' cp.async completions
      mbar_init(o_empty + i, 1 + kKvComputeWarps);  // dV's commit + every compute warp after dS
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kKvComputeWarps);
    mbar_init(p_ready, kKvComputeWarps);
    mbar_init(ds_ready, kKvComputeWarps);
    mbar_init(dv_done, 1);
    mbar_init(dk_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kKvComputeWarps);
    mbar_init(fin, 2);
    unit_ring_init(ring, 2 + kKvComputeWarps);  // both MMA threads and the compute warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kKvMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) {  // scheduler balance record
    if (blockIdx.x == 0) p.cta_times[0] = gridDim.x;
    p.cta_times[1 + 2 * blockIdx.x] = globaltimer_ns();
  }
  const Watchdog wd{p.status, abort_flag, p.timeout_ns};
  const UnitSpace us = unit_space(p.sched, p.Hkv, kSchedKV);
  const int n_units = us.n_units();
  const int G = p.Hq / p.Hkv;

  if (warp == kKvLoadWarp) {
    // ------------------------------------------------------------ loads
    uint32_t t = 0;  // query tiles loaded so far
    int unit_i = 0;
    bool ok = true;
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_produce_warp(ring, us, p.cu, p.sched.next, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      const KvItem it = kv_decode(un);
      if (unit_i > 0 && !warp_wait(kv_empty, (unit_i - 1) & 1, wd, 21)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
        for (int b = 0; b < C::kNumBox; ++b) {
          tma_load_3d(sK + b * C::kBoxBytes, &tm_k, kv_full, 64 * b, it.g, it.k0);
          tma_load_3d(sV + b * C::kBoxBytes, &tm_v, kv_full, 64 * b, it.g, it.k0);
        }
      }
      for (int h = it.g * G; h < (it.g + 1) * G && ok; ++h) {
        for (int m = it.v; m < it.nq; ++m, ++t) {
          const int qs = t % C::kQStages, os = t % C::kOStages;
          const uint32_t qu = t / C::kQStages, ou = t / C::kOStages;
          const int q0 = it.s + 128 * m;
          if (qu > 0 && !warp_wait(q_empty + qs, (qu - 1) & 1, wd, 22)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(q_full + qs, C::kTileBytes);
            for (int b = 0; b < C::kNumBox; ++b)
              tma_load_3d(sQr + qs * C::kTileBytes + b * C::kBoxBytes, &tm_q, q_full + qs, 64 * b, h, q0);
          }
          if (ou > 0 && !warp_wait(o_empty + os, (ou - 1) & 1, wd, 20)) { ok = false; break; }
          uint8_t* ob = sOr + os * C::kOStageBytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(o_full + os, C::kTileBytes);
            for (int b = 0; b < C::kNumBox; ++b)
              tma_load_3d(ob + b * C::kBoxBytes, &tm_do, o_full + os, 64 * b, h, q0);
          }
          // -LSE log2(e) and D of the tile's 128 queries (zeros past the tensor end)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int c = 4 * lane + r, i = q0 + c;
            const bool in = i < p.T;
            const size_t off = in ? (size_t)h * p.T + i : 0;
            cp_async_4(ob + C::kNl2Off + 4 * c, p.nl2 + off, in ? 4 : 0);
            cp_async_4(ob + C::kDeltaOff + 4 * c, p.delta + off, in ? 4 : 0);
          }
          cp_async_mbar_arrive(o_full + os);
        }
      }
    }
    if (lane == 0) {
      // teardown: let this warp's copies land before the CTA exits
      if (unit_i > 0) drain_wait(kv_full, (unit_i - 1) & 1, p.timeout_ns);
      for (uint32_t i = (t > C::kQStages ? t - C::kQStages : 0); i < t; ++i)
        drain_wait(q_full + (i % C::kQStages), (i / C::kQStages) & 1, p.timeout_ns);
      for (uint32_t i = (t > C::kOStages ? t - C::kOStages : 0); i < t; ++i)
        drain_wait(o_full + (i % C::kOStages), (i / C::kOStages) & 1, p.timeout_ns);
    }
  } else if (warp == kKvMmaWarp) {
    // ------------------------------------------------------------ MMA: S^T, dP^T
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, false, false);  // K-major x K-major
      const uint32_t sqr = smem_u32(sQr), sor = smem_u32(sOr);
      // descriptors: base + (byte offset >> 4) in the start-address field
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024), dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
      uint32_t t = 0, s_uses = 0;  // query tiles started; uses of the S^T / dP^T region
      int unit_i = 0;
      bool ok = true;
      // S^T (kv = 0) or dP^T (kv = 1) of tile tt into the region, once the
      // compute warps have read out its previous use
      auto score = [&](uint32_t tt, int kv) {
        if (kv == 0 && !mbar_wait(q_full + (tt % C::kQStages), (tt / C::kQStages) & 1, wd, 26)) return false;
        if (kv == 1 && !mbar_wait(o_full + (tt % C::kOStages), (tt / C::kOStages) & 1, wd, 28)) return false;
        if (s_uses > 0 && !mbar_wait(s_free, (s_uses - 1) & 1, wd, 25)) return false;
        tc_fence_after();
        const uint32_t b_op = kv ? sor + (tt % C::kOStages) * C::kOStageBytes : sqr + (tt % C::kQStages) * C::kTileBytes;
        const uint64_t da = kv ? dv0 : dk0, db = sdesc_sw128(b_op, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
          mma_f16_ss(tmem + C::kSD, da + o, db + o, idesc_s, kk > 0);
        }
        tc_commit(s_full);
        ++s_uses;
        return true;
      };
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const KvItem it = kv_decode(un);
        const int R = G * (it.nq - it.v);
        if (!mbar_wait(kv_full, unit_i & 1, wd, 23)) break;
        for (int r = 0; r < R; ++r, ++t) {
          if (!score(t, 0) || !score(t, 1)) { ok = false; break; }
        }
        if (!ok) break;
        tc_commit(kv_empty);  // K and V are read by these MMAs only
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp == kKvGradWarp) {
    // ------------------------------------------------------------ MMA: dV, dK
    // Q and dO of a tile are released here: the score MMAs that also read them
    // completed before the compute warps signalled P^T (S^T) and dS^T (dP^T).
    if (lane == 0) {
      constexpr uint32_t idesc_g = idesc_f16_f32(128, D, false, true);  // TMEM A x MN-major B
      const uint32_t sqr = smem_u32(sQr), sor = smem_u32(sOr);
      uint32_t t = 0;
      int unit_i = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const KvItem it = kv_decode(un);
        const int R = G * (it.nq - it.v);
        for (int r = 0; r < R; ++r, ++t) {
          const int qs = t % C::kQStages, os = t % C::kOStages;
          // dV += P^T dO
          if (r == 0 && unit_i > 0 && !mbar_wait(acc_free, (unit_i - 1) & 1, wd, 24)) { ok = false; break; }
          if (!mbar_wait(o_full + os, (t / C::kOStages) & 1, wd, 45)) { ok = false; break; }
          if (!mbar_wait(p_ready, t & 1, wd, 27)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ddo = sdesc_sw128(sor + os * C::kOStageBytes, C::kBoxBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(tmem + C::kDV, tmem + C::kP + 8 * kk, ddo + ((kk * 2048) >> 4), idesc_g,
                       (r > 0 || kk > 0) ? 1u : 0u);
          tc_commit(dv_done);
          tc_commit(o_empty + os);
          // dK += dS^T Q
          if (!mbar_wait(q_full + qs, (t / C::kQStages) & 1, wd, 46)) { ok = false; break; }
          if (!mbar_wait(ds_ready, t & 1, wd, 29)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dq = sdesc_sw128(sqr + qs * C::kTileBytes, C::kBoxBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(tmem + C::kDK, tmem + C::kDS + 8 * kk, dq + ((kk * 2048) >> 4), idesc_g,
                       (r > 0 || kk > 0) ? 1u : 0u);
          tc_commit(dk_done);
          tc_commit(q_empty + qs);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row of the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t sd_addr = lane_base + C::kSD + 32 * wg;  // this warpgroup's 32 query columns
    uint32_t t = 0, s_cnt = 0;
    int unit_i = 0;
    bool ok = true;
    auto take = [&](float (&x)[32]) {
      if (!warp_wait(s_full, s_cnt & 1, wd, 30)) return false;
      ++s_cnt;
      tc_fence_after();
      ld_row32(sd_addr, x);
      tc_fence_before();
      warp_arrive(s_free);
      return true;
    };
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      const KvItem it = kv_decode(un);
      const int j = it.k0 + row;  // key index
      for (int h = it.g * G; h < (it.g + 1) * G && ok; ++h) {
        for (int m = it.v; m < it.nq; ++m, ++t) {
          const int os = t % C::kOStages;
          // -LSE log2(e) and D came with the dO stage: wait for the stage itself
          if (!warp_wait(o_full + os, (t / C::kOStages) & 1, wd, 31)) { ok = false; break; }
          const uint8_t* sb = sOr + os * C::kOStageBytes;
          const float* nl2 = reinterpret_cast<const float*>(sb + C::kNl2Off) + 32 * wg;
          const float* dl = reinterpret_cast<const float*>(sb + C::kDeltaOff) + 32 * wg;
          // visible iff j <= i < e; only the diagonal and the last query tile need the test
          const bool full = (m > it.v) && (it.s + 128 * m + 128 <= it.e);
          const int i0 = it.s + 128 * m + 32 * wg;  // query index of this thread's column 0
          // ---- P
          float x[32];
          if (!take(x)) { ok = false; break; }
          {
            // P = 2^(S scale log2(e) - LSE log2(e)): one packed FMA per pair
            const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 n4 = *reinterpret_cast<const float4*>(nl2 + c);
              f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), sl2, f2_pack(n4.x, n4.y)), x[c], x[c + 1]);
              f2_unpack(f2_fma(f2_pack(x[c + 2], x[c + 3]), sl2, f2_pack(n4.z, n4.w)), x[c + 2], x[c + 3]);
#pragma unroll
              for (int u = 0; u < 4; ++u) x[c + u] = fast_exp2(x[c + u]);
            }
          }
          if (!full) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int i = i0 + c;
              if (i < j || i >= it.e) x[c] = 0.f;
            }
          }
          {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) pk[c] = pack_f16x2(x[2 * c], x[2 * c + 1]);
            if (t > 0 && !warp_wait(dv_done, (t - 1) & 1, wd, 32)) { ok = false; break; }
            tc_fence_after();
            tmem_st16(lane_base + C::kP + 16 * wg, pk);
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(p_ready);
          }
          // ---- dS = P (dP - D)
          float y[32];
          if (!take(y)) { ok = false; break; }
          float dm[4] = {0.f, 0.f, 0.f, 0.f};  // range check in four partial chains
          uint32_t dk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            // dS = P (dP - D), packed pairs
            const float4 d4 = *reinterpret_cast<const float4*>(dl + c);
            f2_unpack(f2_mul(f2_pack(x[c], x[c + 1]), f2_sub(f2_pack(y[c], y[c + 1]), f2_pack(d4.x, d4.y))), y[c],
                      y[c + 1]);
            f2_unpack(f2_mul(f2_pack(x[c + 2], x[c + 3]), f2_sub(f2_pack(y[c + 2], y[c + 3]), f2_pack(d4.z, d4.w))),
                      y[c + 2], y[c + 3]);
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            dm[c & 3] = fmaxf(dm[c & 3], fmaxf(fabsf(y[2 * c]), fabsf(y[2 * c + 1])));
            dk[c] = pack_f16x2(y[2 * c], y[2 * c + 1]);
          }
          const float dmax = fmaxf(fmaxf(dm[0], dm[1]), fmaxf(dm[2], dm[3]));
          if (!(dmax < kF16Max)) record_error(p.status, kStatusRange, 42);
          warp_arrive(o_empty + os);  // done with this tile's -LSE log2(e) and D
          if (t > 0 && !warp_wait(dk_done, (t - 1) & 1, wd, 33)) { ok = false; break; }
          tc_fence_after();
          tmem_st16(lane_base + C::kDS + 16 * wg, dk);
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(ds_ready);
        }
      }
      if (!ok) break;
      // epilogue: warpgroups 0, 1 write halves of dV, warpgroups 2, 3 halves of dK * scale
      if (!warp_wait(acc_full, unit_i & 1, wd, 34)) break;
      tc_fence_after();
      const bool valid = j < it.e;
      const bool is_k = wg >= 2;
      const int c0 = (wg & 1) * (D / 2);
      const uint32_t acc_addr = lane_base + (is_k ? C::kDK : C::kDV) + c0;
      void* out = is_k ? p.out0 : p.out1;
      const float mul = is_k ? p.scale : 1.f;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t tt[32];
        tmem_ld32(acc_addr + 32 * c, tt);
        tmem_wait_ld(tt);
        if (valid) store_row32(out, ((size_t)j * p.Hkv + it.g) * D + c0 + 32 * c, tt, mul, p.grad_bf16, p.wide);
      }
      tc_fence_before();
      warp_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kKvMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// 3. dQ
// ---------------------------------------------------------------------------
// TMEM holds dQ, S, dP and the tile's dS (fp16).  The compute warps read S and
// dP out into registers and release them at once, so S and dP of key tile
// v + 1 are computed while dS of tile v is formed; dQ += dS K takes dS from
// TMEM.  Warp 17 issues the score MMAs S and dP, warp 18 the gradient MMA dQ,
// so that a wait of one never leaves the tensor pipe without the other's
// queued work.  16 compute warps: warpgroup wg owns key columns
// [32 wg, 32 wg + 32) of every tile; each thread owns one query row.
constexpr int kQThreads = 608;
constexpr int kQLoadWarp = 16;
constexpr int kQMmaWarp = 17;   // S, dP; owns the TMEM allocation
constexpr int kQGradWarp = 18;  // dQ
constexpr int kQComputeWarps = 16;

template <int D>
struct QCfg : Geo<D> {
  // K and V stream through separate rings: V is released as soon as dP has
  // read it, K only after dQ, so K gets one stage more
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kSmemTiles = (2 + kKStages + kVStages) * Geo<D>::kTileBytes;  // Q, dO, K ring, V ring
  // TMEM: dQ [0,D), S [128,256), dP [256,384), dS [384,448)
  static constexpr uint32_t kDQ = 0, kS = 128, kDP = 256, kDS = 384;
  // bars: q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full, s_free, dp_full, dp_free,
  //       ds_ready, dq_done, acc_full, acc_free, fin
  // + the unit ring's full[8] and empty[8]
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 9 + 2 * kUnitRing;
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
};
static_assert(QCfg<128>::kSmemBytes <= 227 * 1024 && QCfg<64>::kSmemBytes <= 227 * 1024,
              "shared memory of the dQ kernel exceeds the 227 KB a CTA may use");

struct QItem {
  int s, e, m, h, g, q0;  // key tiles 0..m
};

__device__ __forceinline__ QItem q_decode(const BwdParams& p, const UnitInfo& un) {
  QItem it;
  it.m = un.tile;
  it.h = un.h;
  it.g = it.h / (p.Hq / p.Hkv);
  it.s = un.s;
  it.e = un.e;
  it.q0 = it.s + 128 * it.m;
  return it;
}

template <int D>
__global__ void __launch_bounds__(kQThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdParams p) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::kTileBytes;
  uint8_t* sKr = smem + 2 * C::kTileBytes;                  // K ring
  uint8_t* sVr = sKr + C::kKStages * C::kTileBytes;          // V ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_full + 2;
  uint64_t* dp_free = s_full + 3;
  uint64_t* ds_ready = s_full + 4;
  uint64_t* dq_done = s_full + 5;
  uint64_t* acc_full = s_full + 6;
  uint64_t* acc_free = s_full + 7;
  uint64_t* fin = s_full + 8;
  const UnitRing ring{reinterpret_cast<int*>(bars + C::kNumBars) + 4, bars + C::kNumBars - 2 * kUnitRing,
                      bars + C::kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::kKStages; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::kVStages; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kQComputeWarps);
    mbar_init(dp_full, 1);
    mbar_init(dp_free, kQComputeWarps);
    mbar_init(ds_ready, kQComputeWarps);
    mbar_init(dq_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kQComputeWarps);
    mbar_init(fin, 2);
    unit_ring_init(ring, 2 + kQComputeWarps);  // both MMA threads and the compute warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kQMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) {  // scheduler balance record
    if (blockIdx.x == 0) p.cta_times[0] = gridDim.x;
    p.cta_times[1 + 2 * blockIdx.x] = globaltimer_ns();
  }
  const Watchdog wd{p.status, abort_flag, p.timeout_ns};
  const UnitSpace us = unit_space(p.sched, p.Hq, kSchedQ);
  const int n_units = us.n_units();

  if (warp == kQLoadWarp) {
    if (lane == 0) {
      uint32_t kt = 0;  // key tiles loaded (all units)
      int unit_i = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_produce(ring, us, p.cu, p.sched.next, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const QItem it = q_decode(p, un);
        if (unit_i > 0 && !mbar_wait(q_empty, (unit_i - 1) & 1, wd, 31)) break;
        mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
        for (int b = 0; b < C::kNumBox; ++b) {
          tma_load_3d(sQ + b * C::kBoxBytes, &tm_q, q_full, 64 * b, it.h, it.q0);
          tma_load_3d(sDO + b * C::kBoxBytes, &tm_do, q_full, 64 * b, it.h, it.q0);
        }
        for (int v = 0; v <= it.m; ++v, ++kt) {
          const int ks = kt % C::kKStages, vs = kt % C::kVStages;
          const uint32_t ku = kt / C::kKStages, vu = kt / C::kVStages;
          const int k0 = it.s + 128 * v;
          if (ku > 0 && !mbar_wait(k_empty + ks, (ku - 1) & 1, wd, 32)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + ks, C::kTileBytes);
          for (int b = 0; b < C::kNumBox; ++b)
            tma_load_3d(sKr + ks * C::kTileBytes + b * C::kBoxBytes, &tm_k, k_full + ks, 64 * b, it.g, k0);
          if (vu > 0 && !mbar_wait(v_empty + vs, (vu - 1) & 1, wd, 30)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full + vs, C::kTileBytes);
          for (int b = 0; b < C::kNumBox; ++b)
            tma_load_3d(sVr + vs * C::kTileBytes + b * C::kBoxBytes, &tm_v, v_full + vs, 64 * b, it.g, k0);
        }
      }
      if (unit_i > 0) drain_wait(q_full, (unit_i - 1) & 1, p.timeout_ns);
      for (uint32_t i = (kt > C::kKStages ? kt - C::kKStages : 0); i < kt; ++i)
        drain_wait(k_full + (i % C::kKStages), (i / C::kKStages) & 1, p.timeout_ns);
      for (uint32_t i = (kt > C::kVStages ? kt - C::kVStages : 0); i < kt; ++i)
        drain_wait(v_full + (i % C::kVStages), (i / C::kVStages) & 1, p.timeout_ns);
    }
  } else if (warp == kQMmaWarp) {
    // ------------------------------------------------------------ MMA: S, dP
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, false, false);
      const uint32_t skr = smem_u32(sKr), svr = smem_u32(sVr);
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024), ddo0 = sdesc_sw128(smem_u32(sDO), 16, 1024);
      uint32_t kt = 0;  // key tiles started (all units)
      int unit_i = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const QItem it = q_decode(p, un);
        if (!mbar_wait(q_full, unit_i & 1, wd, 33)) break;
        for (int v = 0; v <= it.m; ++v, ++kt) {
          // S and dP of key tile kt into their regions, each once the compute
          // warps have read out its previous use
          const int ks = kt % C::kKStages, vs = kt % C::kVStages;
          if (!mbar_wait(k_full + ks, (kt / C::kKStages) & 1, wd, 35)) { ok = false; break; }
          if (kt > 0 && !mbar_wait(s_free, (kt - 1) & 1, wd, 36)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(skr + ks * C::kTileBytes, 16, 1024);
          const uint64_t dv = sdesc_sw128(svr + vs * C::kTileBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
            mma_f16_ss(tmem + C::kS, dq0 + o, dk + o, idesc_s, kk > 0);
          }
          tc_commit(s_full);
          if (kt > 0 && !mbar_wait(dp_free, (kt - 1) & 1, wd, 37)) { ok = false; break; }
          if (!mbar_wait(v_full + vs, (kt / C::kVStages) & 1, wd, 44)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
            mma_f16_ss(tmem + C::kDP, ddo0 + o, dv + o, idesc_s, kk > 0);
          }
          tc_commit(dp_full);
          tc_commit(v_empty + vs);  // V is read only by dP
        }
        if (!ok) break;
        tc_commit(q_empty);  // Q and dO are read only by S and dP
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp == kQGradWarp) {
    // ------------------------------------------------------------ MMA: dQ
    // K of a tile is released here: S, its other reader, completed before the
    // compute warps signalled dS.
    if (lane == 0) {
      constexpr uint32_t idesc_g = idesc_f16_f32(128, D, false, true);
      const uint32_t skr = smem_u32(sKr);
      uint32_t kt = 0;
      int unit_i = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const QItem it = q_decode(p, un);
        for (int v = 0; v <= it.m; ++v, ++kt) {
          const int ks = kt % C::kKStages;
          if (v == 0 && unit_i > 0 && !mbar_wait(acc_free, (unit_i - 1) & 1, wd, 34)) { ok = false; break; }
          if (!mbar_wait(k_full + ks, (kt / C::kKStages) & 1, wd, 47)) { ok = false; break; }
          if (!mbar_wait(ds_ready, kt & 1, wd, 38)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dkm = sdesc_sw128(skr + ks * C::kTileBytes, C::kBoxBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(tmem + C::kDQ, tmem + C::kDS + 8 * kk, dkm + ((kk * 2048) >> 4), idesc_g,
                       (v > 0 || kk > 0) ? 1u : 0u);
          tc_commit(dq_done);
          tc_commit(k_empty + ks);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else {
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t kt = 0;  // key tiles processed (all units)
    int unit_i = 0;
    bool ok = true;
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      const QItem it = q_decode(p, un);
      const int i = it.q0 + row;
      const bool valid = i < it.e;
      // rows past the document end (the tail of the last tile) get P = 0
      const float nl2 = valid ? p.nl2[(size_t)it.h * p.T + i] : -INFINITY;
      const float dl = valid ? p.delta[(size_t)it.h * p.T + i] : 0.f;
      for (int v = 0; v <= it.m; ++v, ++kt) {
        float x[32], y[32];
        if (!warp_wait(s_full, kt & 1, wd, 39)) { ok = false; break; }
        tc_fence_after();
        ld_row32(lane_base + C::kS + 32 * wg, x);
        tc_fence_before();
        warp_arrive(s_free);
        if (!warp_wait(dp_full, kt & 1, wd, 40)) { ok = false; break; }
        tc_fence_after();
        ld_row32(lane_base + C::kDP + 32 * wg, y);
        tc_fence_before();
        warp_arrive(dp_free);
        const int j0 = it.s + 128 * v + 32 * wg;  // key index of this thread's column 0
        const bool diag = v == it.m;
        uint32_t dk[16];
        float dm[4] = {0.f, 0.f, 0.f, 0.f};  // range check in four partial chains
        const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2), nl22 = f2_pack(nl2, nl2), dl2 = f2_pack(dl, dl);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          // P = 2^(S scale log2(e) - LSE log2(e)), dS = P (dP - D): packed pairs
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), sl2, nl22), a0, a1);
          float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
          if (diag && j0 + c > i) p0 = 0.f;
          if (diag && j0 + c + 1 > i) p1 = 0.f;
          float dv[2];
          f2_unpack(f2_mul(f2_pack(p0, p1), f2_sub(f2_pack(y[c], y[c + 1]), dl2)), dv[0], dv[1]);
          dm[(c / 2) & 3] = fmaxf(dm[(c / 2) & 3], fmaxf(fabsf(dv[0]), fabsf(dv[1])));
          dk[c / 2] = pack_f16x2(dv[0], dv[1]);
        }
        const float dmax = fmaxf(fmaxf(dm[0], dm[1]), fmaxf(dm[2], dm[3]));
        if (!(dmax < kF16Max)) record_error(p.status, kStatusRange, 43);
        if (kt > 0 && !warp_wait(dq_done, (kt - 1) & 1, wd, 41)) { ok = false; break; }
        tc_fence_after();
        tmem_st16(lane_base + C::kDS + 16 * wg, dk);  // dS -> columns [16 wg, 16 wg + 16)
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(ds_ready);
      }
      if (!ok) break;
      if (!warp_wait(acc_full, unit_i & 1, wd, 42)) break;
      tc_fence_after();
      // warpgroup wg writes channels [wg D/4, (wg+1) D/4) of dQ * scale
      if (D == 128 || wg < 2) {
        uint32_t t[32];
        const int col = wg * 32;
        tmem_ld32(lane_base + C::kDQ + col, t);
        tmem_wait_ld(t);
        if (valid) store_row32(p.out0, ((size_t)i * p.Hq + it.h) * D + col, t, p.scale, p.grad_bf16, p.wide);
      }
      tc_fence_before();
      warp_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kQMmaWarp) tmem_dealloc(tmem, 512);
}

template <int D>
cudaError_t launch_d(const BwdArgs& a, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_thd(&tq, a.q16, a.T, a.Hq, D, true) || !make_tmap_thd(&tk, a.k16, a.T, a.Hkv, D, true) ||
      !make_tmap_thd(&tv, a.v16, a.T, a.Hkv, D, true) || !make_tmap_thd(&tdo, a.do16, a.T, a.Hq, D, true))
    return cudaErrorInvalidValue;
  // 1. D
  a.marks.at(3, stream);
  {
    constexpr int rows_per_block = 256 / (D / 8);
    const long long rows = (long long)a.T * a.Hq;
    const unsigned grid = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    delta_kernel<D><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.o_resid),
        static_cast<const __nv_bfloat16*>(a.dout), static_cast<const __nv_bfloat16*>(a.q),
        static_cast<uint4*>(a.do16), static_cast<uint4*>(a.q16), a.lse, a.delta, a.nl2, a.T, a.Hq, a.status);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  BwdParams p;
  p.cu = a.cu;
  p.lse = a.lse;
  p.delta = a.delta;
  p.nl2 = a.nl2;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.grad_bf16 = a.grad_bf16;
  // 2. dK, dV
  a.marks.at(4, stream);
  {
    using C = KvCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    BwdParams pk = p;
    pk.sched = sched_view(a.sched_kv);
    pk.cta_times = a.cta_times[0];
    pk.out0 = a.dk;
    pk.out1 = a.dv;
    pk.wide = aligned32(a.dk) && aligned32(a.dv);
    const long long max_units = (long long)a.sched_kv.max_items * a.Hkv;
    const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
    dkdv_kernel<D><<<grid, kKvThreads, C::kSmemBytes, stream>>>(tq, tk, tv, tdo, pk);
    note_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 3. dQ
  a.marks.at(5, stream);
  {
    using C = QCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    BwdParams pq = p;
    pq.sched = sched_view(a.sched_q);
    pq.cta_times = a.cta_times[1];
    pq.out0 = a.dq;
    pq.wide = aligned32(a.dq);
    pq.out1 = nullptr;
    const long long max_units = (long long)a.sched_q.max_items * a.Hq;
    const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
    dq_kernel<D><<<grid, kQThreads, C::kSmemBytes, stream>>>(tq, tk, tv, tdo, pq);
    note_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  a.marks.at(6, stream);
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

}  // namespace fapk
