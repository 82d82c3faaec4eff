// Backward of causal packed-document attention, MXFP8 path, for sm_100a
// (FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri": MXFP8
// operands with shared E8M0 scales, quantised operands reused across the
// forward and backward orientations, leak guards, fwd/bwd consistency).
//
// The straight-through gradient of the MXFP8 forward, from the same quantised
// operands (the forward's ctx holds Q, K, V in both forms; dO is quantised
// here):
//   P    = exp(S - LSE), S from Q~pt and K~ (rule L)      D = dO . O
//   dP   = dO~pt V~^T (rule L on V)                        dS = P (dP - D)
//   dQ   = scale dS~ K~   (dS~ per (query row, key block); K by rule L)
//   dK   = scale dS~T Q~tb,  dV = P~T dO~tb   (dS~T, P~T per (key row, query block))
// Rule L on the key side: token-block forms for key blocks before the query's
// block, per-token forms on the diagonal 32x32 blocks.
//
// Two kernels, deterministic (no atomics), both persistent with 1 CTA per SM:
//  * dq_mx:   item = (document, 128-query tile, head); one thread per query
//    row.  Per key tile: S = Q K^T and dP = dO V^T (block-scaled FP8, K and V
//    in token-block form; on the diagonal tile a second phase with the
//    per-token forms into the same TMEM columns), dS~ quantised into shared
//    memory, dQ += dS~ K~tb (FP8, the same K~tb bytes read MN-major) plus, on
//    the diagonal tile, the diagonal blocks as an exact bf16 MMA with the
//    per-token K, which the compute warps dequantise on load at the start of
//    each item.
//  * dkdv_mx: item = (document, 128-key tile, KV head); one thread per key
//    row, warpgroup w on query columns [64w, 64w + 64).  Per query tile:
//    S^T then dP^T into one TMEM region in turn (TMEM also holds dV, dK and
//    the scale factors), P~T and dS~T quantised into shared memory,
//    dV += P~T dO~tb and dK += dS~T Q~tb as block-scaled FP8 MMAs.
//
// Mixed NVFP4/FP8 path (kNv): the scores are recomputed from the forward's
// NVFP4 Q and K (kind::mxf4nvf4, two MMAs of K = 64 per tile), the same
// product the forward took; the diagonal tile's second score phase repeats
// it on the same tiles (NVFP4 blocks never pool tokens), so the compute
// warps run unchanged.  dP and the gradient products are the MXFP8 path's.
#include <cuda_bf16.h>

#include "internal.h"
#include "mx.cuh"
#include "nv.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace fapk {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCode = 128 * 128;      // 128 rows x 128 fp8 codes
constexpr int kBf16 = 128 * 128 * 2;  // 128 rows x 128 bf16
constexpr int kBox = 128 * 64 * 2;    // one 64-element bf16 box of 128 rows
constexpr int kSfBlk = 512;

// Scale block of an MN-major operand whose rows are the 128 channels and
// whose K blocks are the token blocks blk0..blk0+3 (token-block form): byte
// kb of the word of channel row (lane + 32 r1) is the scale of (block
// blk0 + kb, channel group r1).
__device__ __forceinline__ uint4 tb_channel_rows(const uint8_t* stb, int s, int e, int doc, int blk0, int H, int g) {
  uint32_t wv[4] = {0, 0, 0, 0};
#pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    const uint32_t t = tb_word(stb, s, e, doc, blk0 + kb, H, g);
#pragma unroll
    for (int r1 = 0; r1 < 4; ++r1) wv[r1] |= ((t >> (8 * r1)) & 0xFFu) << (8 * kb);
  }
  return make_uint4(wv[0], wv[1], wv[2], wv[3]);
}

__device__ __forceinline__ uint4 pt_rows(const uint8_t* spt, int t0, int lane, int T, int H, int h) {
  return make_uint4(pt_word(spt, t0 + lane, T, H, h), pt_word(spt, t0 + lane + 32, T, H, h),
                    pt_word(spt, t0 + lane + 64, T, H, h), pt_word(spt, t0 + lane + 96, T, H, h));
}

__device__ __forceinline__ uint4 tb_rows(const uint8_t* stb, int s, int e, int doc, int blk0, int H, int g) {
  return make_uint4(tb_word(stb, s, e, doc, blk0, H, g), tb_word(stb, s, e, doc, blk0 + 1, H, g),
                    tb_word(stb, s, e, doc, blk0 + 2, H, g), tb_word(stb, s, e, doc, blk0 + 3, H, g));
}

// MX quantisation of 32 values (one block of a computed operand): 8 code
// words; returns the scale byte.  A value that rounds to zero from below keeps
// the code 0x80 (-0), which adds nothing to an MMA.
__device__ __forceinline__ uint32_t quant32(const float (&x)[32], int rule, uint32_t (&codes)[8]) {
  float m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = max_abs_xs(x[k], x[4 + k]);
#pragma unroll
  for (int c = 8; c < 32; c += 4) {
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = max_abs_xs(m[k], x[c + k]);
  }
  const float amax = fabsf(max_abs_xs(max_abs_xs(m[0], m[1]), max_abs_xs(m[2], m[3])));
  const int X = mx_block_exponent(amax, rule);
  const float sc = mx_pow2_neg(X < -126 ? -126 : X);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    codes[c] = mx_e4m3x2(x[4 * c] * sc, x[4 * c + 1] * sc) | (mx_e4m3x2(x[4 * c + 2] * sc, x[4 * c + 3] * sc) << 16);
  return (uint32_t)(X + 127);
}

// Exact bf16 of the dequantised block: 16 words of packed bf16 pairs.
__device__ __forceinline__ void dequant32_bf16(const uint32_t (&codes)[8], uint32_t sbyte, uint32_t (&out)[16]) {
  const int X = (int)sbyte - 127;
  const float sc = mx_pow2(X < -126 ? -126 : X);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float a, b, cc, d;
    mx_decode2(codes[c] & 0xFFFFu, a, b);
    mx_decode2(codes[c] >> 16, cc, d);
    out[2 * c] = pack_bf16x2(a * sc, b * sc);
    out[2 * c + 1] = pack_bf16x2(cc * sc, d * sc);
  }
}

// 8 code words (32 codes) into row `row` of a K-major FP8 tile at 16-byte
// chunks c0, c0+1 (128-byte swizzle).
__device__ __forceinline__ void store_codes32(uint8_t* tile, int row, int c0, const uint32_t (&w)[8]) {
  uint8_t* prow = tile + row * 128;
  *reinterpret_cast<uint4*>(prow + ((c0 ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(prow + (((c0 + 1) ^ (row & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
}

// 32 bf16 (16 words) into row `row` of a K-major bf16 tile (two 64-element
// boxes) at element offset 32 q (q = 0..3).
__device__ __forceinline__ void store_bf16_32(uint8_t* tile, int row, int q, const uint32_t (&w)[16]) {
  const int box = q >> 1, c0 = (q & 1) * 4;
  uint8_t* prow = tile + box * kBox + row * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(prow + (((c0 + c) ^ (row & 7)) << 4)) =
        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

struct MxParams {
  const int32_t* cu;
  SchedView sched;
  const float* lse;
  const float* delta;
  const uint8_t *q_stb, *q_spt, *k_stb, *k_spt, *v_stb, *v_spt, *do_stb, *do_spt;
  const uint8_t *q_nvs, *k_nvs;  // mixed path: NVFP4 scales of Q [T][Hq][8] and K [T][Hkv][8]
  const uint8_t* k_vpt;          // mixed path: K per-token codes (dQ's diagonal, read directly)
  void* out0;  // dq | dk
  void* out1;  // -  | dv
  DeviceStatus* status;
  uint64_t timeout_ns;
  int T, Hq, Hkv;
  int d;  // head dimension of the bf16/fp32 tensors (64 or 128); the codes always have 128 per row
  float scale, scale_log2;
  int grad_bf16;
  int wide;  // every gradient output 32-byte aligned: 32-byte stores
  int rule;
  unsigned long long* cta_times;  // per-CTA (start, end) records, or null
};

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
namespace dqk {
// warps 0-15: one thread per (query row, 32-key block): warpgroup wg on key
// block wg of every tile (one MX scale block of dS~); warp 16: loads; warp 17:
// the score MMAs S and dP; warp 18: the dQ MMAs (two issuing threads, so that a
// wait of one never leaves the tensor pipe without the other's queued work)
constexpr int kThreads = 608, kLoad = 16, kMma = 17, kGrad = 18, kComputeWarps = 16, kStages = 2;
constexpr int oQ = 0, oDO = oQ + kCode, oRing = oDO + kCode;  // ring stage: K^tb, V^tb codes
constexpr int oKpt = oRing + kStages * 2 * kCode, oVpt = oKpt + kCode, oKd = oVpt + kCode;  // diag
constexpr int oDS = oKd + kBf16, oDSd = oDS + kCode;
constexpr int oSf = oDSd + kBf16;  // sfQ, sfDO, sfKpt, sfVpt, sfDS, per stage {sfK, sfV, sfKdq}
// mixed path: the NVFP4 K tile of stage s at oKpt + s kNvTile (the per-token K
// tile is not loaded: its dequantised copy is read from global memory); Q's
// second scale block in the sfKpt slot, stage s's second K block at 5 + 3 kStages + s
constexpr int kNvTile = 128 * 64;
constexpr int kNumSf = 5 + 4 * kStages;
constexpr int oBars = oSf + kNumSf * kSfBlk;
// bars: q_full, q_empty, st_full[S], st_empty[S], s_full, s_free, dp_full, dp_free, ds_ready, dq_done,
//       acc_full, acc_free, fin, kd_full
// + the unit ring's full[8] and empty[8]
constexpr int kNumBars = 2 + 2 * kStages + 10 + 2 * kUnitRing;
constexpr int kSmem = oBars + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory exceeds the 227 KB a CTA may use");
// TMEM: S and dP regions (each read out into registers and released at
// once), dQ, scale factors
constexpr uint32_t tS = 0, tDP = 128, tDQ = 256;
constexpr uint32_t tSfQ = 384, tSfDO = 388, tSfK = 392, tSfV = 396, tSfKpt = 400, tSfVpt = 404, tSfDS = 408,
                   tSfKdq = 412, tSfK2 = 416;  // mixed path: tSfKpt holds Q's second block, tSfK2 K's
constexpr uint32_t kSfCols[] = {tSfQ, tSfDO, tSfK, tSfV, tSfKpt, tSfVpt, tSfDS, tSfKdq, tSfK2};
static_assert(sf_cols_ok(kSfCols, tDQ + 128), "dQ kernel TMEM scale columns overlap");
}  // namespace dqk

// kNv: tm_qpt maps Q's NVFP4 codes, tm_knv K's (tm_kpt is not read)
template <bool kNv>
__global__ void __launch_bounds__(dqk::kThreads, 1)
    dq_mx_kernel(const __grid_constant__ CUtensorMap tm_qpt, const __grid_constant__ CUtensorMap tm_dopt,
                 const __grid_constant__ CUtensorMap tm_ktb, const __grid_constant__ CUtensorMap tm_vtb,
                 const __grid_constant__ CUtensorMap tm_kpt, const __grid_constant__ CUtensorMap tm_vpt,
                 const __grid_constant__ CUtensorMap tm_knv, const MxParams p) {
  using namespace dqk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sf = smem + oSf;  // 512-byte scale blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* st_empty = bars + 2 + kStages;
  uint64_t* s_full = bars + 2 + 2 * kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_full + 2;
  uint64_t* dp_free = s_full + 3;
  uint64_t* ds_ready = s_full + 4;
  uint64_t* dq_done = s_full + 5;
  uint64_t* acc_full = s_full + 6;
  uint64_t* acc_free = s_full + 7;
  uint64_t* fin = s_full + 8;
  uint64_t* kd_full = s_full + 9;  // the diagonal per-token K dequantised to bf16 (compute warps)
  const UnitRing ring{reinterpret_cast<int*>(bars + kNumBars) + 4, bars + kNumBars - 2 * kUnitRing,
                      bars + kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto sfb = [&](int i) { return sf + i * kSfBlk; };  // 0 Q, 1 dO, 2 Kpt, 3 Vpt, 4 dS, 5+3s+{0,1,2} stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 32);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(st_full + i, 32);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kComputeWarps);
    mbar_init(dp_full, 1);
    mbar_init(dp_free, kComputeWarps);
    mbar_init(ds_ready, kComputeWarps);
    mbar_init(dq_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kComputeWarps);
    mbar_init(fin, 2);
    mbar_init(kd_full, kComputeWarps);
    unit_ring_init(ring, 2 + kComputeWarps);  // both MMA threads and the compute warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMma) {
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
  auto decode = [&](const UnitInfo& un, int& doc, int& s, int& e, int& h, int& g, int& q0, int& n) {
    const int m = un.tile;
    doc = un.doc;
    h = un.h;
    g = h / (p.Hq / p.Hkv);
    s = un.s;
    e = un.e;
    q0 = s + 128 * m;
    n = m + 1;
  };

  if (warp == kLoad) {
    uint32_t st_it = 0;
    int unit_i = 0;
    bool ok = true;
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_produce_warp(ring, us, p.cu, p.sched.next, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      int doc, s, e, h, g, q0, n;
      decode(un, doc, s, e, h, g, q0, n);
      // the scale words' global reads first, so that their latency overlaps the wait
      uint4 w_0, w_2;
      if constexpr (kNv) {
        const uint2 w0 = nv_scale_words(p.q_nvs, q0 + lane, p.T, p.Hq, h);
        const uint2 w1 = nv_scale_words(p.q_nvs, q0 + lane + 32, p.T, p.Hq, h);
        const uint2 w2 = nv_scale_words(p.q_nvs, q0 + lane + 64, p.T, p.Hq, h);
        const uint2 w3 = nv_scale_words(p.q_nvs, q0 + lane + 96, p.T, p.Hq, h);
        w_0 = make_uint4(w0.x, w1.x, w2.x, w3.x);
        w_2 = make_uint4(w0.y, w1.y, w2.y, w3.y);
      } else {
        w_0 = pt_rows(p.q_spt, q0, lane, p.T, p.Hq, h);
        w_2 = pt_rows(p.k_spt, q0, lane, p.T, p.Hkv, g);
      }
      const uint4 w_1 = pt_rows(p.do_spt, q0, lane, p.T, p.Hq, h);
      const uint4 w_3 = pt_rows(p.v_spt, q0, lane, p.T, p.Hkv, g);
      if (unit_i > 0 && !warp_wait(q_empty, (unit_i - 1) & 1, wd, 71)) break;
      reinterpret_cast<uint4*>(sfb(0))[lane] = w_0;
      reinterpret_cast<uint4*>(sfb(1))[lane] = w_1;
      reinterpret_cast<uint4*>(sfb(2))[lane] = w_2;
      reinterpret_cast<uint4*>(sfb(3))[lane] = w_3;
      fence_proxy_async_smem();
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, kNv ? kNvTile + 2 * kCode : 4 * kCode);
        tma_load_3d(smem + oQ, &tm_qpt, q_full, 0, h, q0);
        tma_load_3d(smem + oDO, &tm_dopt, q_full, 0, h, q0);
        if (!kNv) tma_load_3d(smem + oKpt, &tm_kpt, q_full, 0, g, q0);  // the diagonal key tile starts at q0
        tma_load_3d(smem + oVpt, &tm_vpt, q_full, 0, g, q0);
      } else {
        mbar_arrive(q_full);
      }
      for (int v = 0; v < n; ++v, ++st_it) {
        const int stg = st_it % kStages;
        const uint32_t use = st_it / kStages;
        // scale words first, so that their global reads overlap the wait
        uint4 wk, wk2 = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (kNv) {
          // the NVFP4 scale words of the tile's keys (scores)
          const int k0 = s + 128 * v;
          const uint2 w0 = nv_scale_words(p.k_nvs, k0 + lane, p.T, p.Hkv, g);
          const uint2 w1 = nv_scale_words(p.k_nvs, k0 + lane + 32, p.T, p.Hkv, g);
          const uint2 w2 = nv_scale_words(p.k_nvs, k0 + lane + 64, p.T, p.Hkv, g);
          const uint2 w3 = nv_scale_words(p.k_nvs, k0 + lane + 96, p.T, p.Hkv, g);
          wk = make_uint4(w0.x, w1.x, w2.x, w3.x);
          wk2 = make_uint4(w0.y, w1.y, w2.y, w3.y);
        } else {
          wk = tb_rows(p.k_stb, s, e, doc, 4 * v, p.Hkv, g);
        }
        const uint4 wv = tb_rows(p.v_stb, s, e, doc, 4 * v, p.Hkv, g);
        const uint4 wkc = tb_channel_rows(p.k_stb, s, e, doc, 4 * v, p.Hkv, g);
        if (use > 0 && !warp_wait(st_empty + stg, (use - 1) & 1, wd, 72)) { ok = false; break; }
        reinterpret_cast<uint4*>(sfb(5 + 3 * stg))[lane] = wk;
        reinterpret_cast<uint4*>(sfb(6 + 3 * stg))[lane] = wv;
        reinterpret_cast<uint4*>(sfb(7 + 3 * stg))[lane] = wkc;
        if (kNv) reinterpret_cast<uint4*>(sfb(5 + 3 * kStages + stg))[lane] = wk2;
        fence_proxy_async_smem();
        if (lane == 0) {
          uint8_t* st = smem + oRing + stg * 2 * kCode;
          mbar_arrive_expect_tx(st_full + stg, kNv ? 2 * kCode + kNvTile : 2 * kCode);
          tma_load_3d(st, &tm_ktb, st_full + stg, 0, g, s + 128 * v);
          tma_load_3d(st + kCode, &tm_vtb, st_full + stg, 0, g, s + 128 * v);
          if (kNv) tma_load_3d(smem + oKpt + stg * kNvTile, &tm_knv, st_full + stg, 0, g, s + 128 * v);
        } else {
          mbar_arrive(st_full + stg);
        }
      }
    }
    if (lane == 0) {
      if (unit_i > 0) drain_wait(q_full, (unit_i - 1) & 1, p.timeout_ns);
      for (uint32_t i = (st_it > kStages ? st_it - kStages : 0); i < st_it; ++i)
        drain_wait(st_full + (i % kStages), (i / kStages) & 1, p.timeout_ns);
    }
  } else if (warp == kMma || warp == kGrad) {
    if (lane == 0) {
      const uint32_t aQ = smem_u32(smem + oQ), aDO = smem_u32(smem + oDO), aRing = smem_u32(smem + oRing),
                     aKpt = smem_u32(smem + oKpt), aVpt = smem_u32(smem + oVpt), aKd = smem_u32(smem + oKd),
                     aDS = smem_u32(smem + oDS), aDSd = smem_u32(smem + oDSd), aSf = smem_u32(sf);
      uint32_t kt = 0, s_uses = 0, dp_uses = 0;
      int unit_i = 0;
      bool ok = true;
      // D (tmem col) = A B^T, both K-major codes, block scales at TMEM cols sfa/sfb
      auto mx_kk = [&](uint32_t dcol, uint32_t a, uint32_t b, uint32_t sfa, uint32_t sfbc, bool b_mn,
                       bool acc_first) {
        const uint64_t da = sdesc_sw128(a, 16, 1024), db = b_mn ? sdesc_sw128(b, 16384, 1024) : sdesc_sw128(b, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_mxf8_ss(tmem + dcol, da + ((kk * 32) >> 4), db + ((b_mn ? kk * 4096 : kk * 32) >> 4),
                      idesc_mxf8(128, 128, b_mn, kk, kk), (tmem + sfa) | ((uint32_t)kk << 30),
                      (tmem + sfbc) | ((uint32_t)kk << 30), (acc_first || kk > 0) ? 1u : 0u);
      };
      if (warp == kMma) {
        // ---------------------------------------------- S, dP
        // each score MMA goes into its region once the compute warps have read
        // out the previous use; the regions' reads of Q, dO, the per-token K and
        // V and the stage's V end here, K^tb is read by dQ too
        // (mixed path: S from the NVFP4 Q and the stage's NVFP4 K, whose
        // second scale blocks sit at tSfKpt and tSfK2)
        // (a stage's K or V scale block is copied into TMEM only after the
        // region's previous MMA, which read the same scale columns, has been
        // read out, i.e. has completed; cp_src 0: no copy)
        auto score = [&](bool dp, uint32_t a, uint32_t b, uint32_t sfa, uint32_t sfbc, uint32_t cp_src = 0,
                         uint32_t cp_src2 = 0) {
          uint32_t& uses = dp ? dp_uses : s_uses;
          if (uses > 0 && !mbar_wait(dp ? dp_free : s_free, (uses - 1) & 1, wd, dp ? 74 : 73)) return false;
          tc_fence_after();
          if (cp_src) tmem_cp_sf(tmem + sfbc, cp_src);
          if (cp_src2) tmem_cp_sf(tmem + tSfK2, cp_src2);
          if (kNv && !dp) {
            const uint64_t da = sdesc_sw64(a), db = sdesc_sw64(b);
            constexpr uint32_t idn = idesc_nvf4(128, 128);
            mma_nvf4_ss(tmem + tS, da, db, idn, tmem + sfa, tmem + sfbc, 0u);
            mma_nvf4_ss(tmem + tS, da + 2, db + 2, idn, tmem + tSfKpt, tmem + tSfK2, 1u);
          } else {
            mx_kk(dp ? tDP : tS, a, b, sfa, sfbc, false, false);
          }
          tc_commit(dp ? dp_full : s_full);
          ++uses;
          return true;
        };
        for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
          const UnitInfo un = unit_take(ring, uk, wd);
          const int w = un.w;
          if (w < 0 || w >= n_units) break;
          int doc, s, e, h, g, q0, n;
          decode(un, doc, s, e, h, g, q0, n);
          if (!mbar_wait(q_full, unit_i & 1, wd, 76)) break;
          tc_fence_after();
          tmem_cp_sf(tmem + tSfQ, aSf + 0 * kSfBlk);
          tmem_cp_sf(tmem + tSfDO, aSf + 1 * kSfBlk);
          tmem_cp_sf(tmem + tSfKpt, aSf + 2 * kSfBlk);
          tmem_cp_sf(tmem + tSfVpt, aSf + 3 * kSfBlk);
          for (int v = 0; v < n; ++v, ++kt) {
            // token-block S and dP of key tile kt
            const int stg = kt % kStages;
            if (!mbar_wait(st_full + stg, (kt / kStages) & 1, wd, 75)) { ok = false; break; }
            const uint32_t ak = aRing + stg * 2 * kCode, av = ak + kCode;
            if (!score(false, aQ, kNv ? aKpt + stg * kNvTile : ak, tSfQ, tSfK, aSf + (5 + 3 * stg) * kSfBlk,
                       kNv ? aSf + (5 + 3 * kStages + stg) * kSfBlk : 0u)) { ok = false; break; }
            if (!score(true, aDO, av, tSfDO, tSfV, aSf + (6 + 3 * stg) * kSfBlk)) { ok = false; break; }
          }
          if (!ok) break;
          // the diagonal tile again with the per-token K and V (mixed path:
          // the same NVFP4 scores again, from the last stage, which stays
          // loaded until the dQ MMAs of this tile release it)
          const uint32_t s2 = kNv ? aKpt + ((kt - 1) % kStages) * kNvTile : aKpt;
          if (!score(false, aQ, s2, tSfQ, kNv ? tSfK : tSfKpt) || !score(true, aDO, aVpt, tSfDO, tSfVpt)) break;
        }
      } else {
        // ---------------------------------------------- dQ
        // the stage and the unit's buffers are released here: the score MMAs
        // that also read them completed before the compute warps signalled dS~
        for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
          const UnitInfo un = unit_take(ring, uk, wd);
          const int w = un.w;
          if (w < 0 || w >= n_units) break;
          int doc, s, e, h, g, q0, n;
          decode(un, doc, s, e, h, g, q0, n);
          if (!mbar_wait(q_full, unit_i & 1, wd, 101)) break;
          for (int v = 0; v < n; ++v, ++kt) {
            const int stg = kt % kStages;
            const bool diag = v == n - 1;
            if (v == 0 && unit_i > 0 && !mbar_wait(acc_free, (unit_i - 1) & 1, wd, 77)) { ok = false; break; }
            if (!mbar_wait(st_full + stg, (kt / kStages) & 1, wd, 102)) { ok = false; break; }
            if (!mbar_wait(ds_ready, kt & 1, wd, 78)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ak = aRing + stg * 2 * kCode;
            tmem_cp_sf(tmem + tSfDS, aSf + 4 * kSfBlk);
            tmem_cp_sf(tmem + tSfKdq, aSf + (7 + 3 * stg) * kSfBlk);
            mx_kk(tDQ, aDS, ak, tSfDS, tSfKdq, true, v > 0);
            if (diag) {
              // diagonal 32x32 blocks: exact bf16 dS~ times dequantised per-token K
              if (!mbar_wait(kd_full, unit_i & 1, wd, 103)) { ok = false; break; }
              tc_fence_after();
              constexpr uint32_t idesc_d = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_f16_ss(tmem + tDQ, sdesc_sw128(aDSd + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024),
                           sdesc_sw128(aKd + kk * 2048, kBox, 1024), idesc_d, 1u);
            }
            tc_commit(dq_done);
            tc_commit(st_empty + stg);
          }
          if (!ok) break;
          tc_commit(acc_full);
          tc_commit(q_empty);
        }
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp < kComputeWarps) {
    // one thread per (query row, key block wg)
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lb = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sDS = smem + oDS;
    uint8_t* sDSd = smem + oDSd;
    uint8_t* sfDS = sfb(4);
    uint32_t s_cnt = 0, dp_cnt = 0, kt = 0;
    int unit_i = 0;
    bool ok = true;
    auto take = [&](uint64_t* full, uint64_t* free_bar, uint32_t& cnt, uint32_t col, bool load, uint32_t (&r)[32]) {
      if (!warp_wait(full, cnt & 1, wd, 79)) return false;
      ++cnt;
      tc_fence_after();
      if (load) {
        tmem_ld32(lb + col + 32 * wg, r);
        tmem_wait_ld(r);
      }
      tc_fence_before();
      warp_arrive(free_bar);
      return true;
    };
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      int doc, s, e, h, g, q0, n;
      decode(un, doc, s, e, h, g, q0, n);
      const int i = q0 + row;
      const bool valid = i < e;
      {
        // the diagonal per-token K, dequantised to bf16 for the exact
        // diagonal-block product: this thread's key row `row`, channels
        // 32 wg .. 32 wg + 31.  The previous item's dQ MMAs have completed
        // (q_full of this item follows the loader's wait on q_empty).
        if (!warp_wait(q_full, unit_i & 1, wd, 104)) break;
        uint4 c0, c1;
        uint32_t ksb;
        if constexpr (kNv) {
          // (mixed path: from global memory; the shared tile holds NVFP4 K)
          const int t = q0 + row;
          c0 = c1 = make_uint4(0u, 0u, 0u, 0u);
          ksb = 127u;
          if (t < p.T) {
            const uint4* src = reinterpret_cast<const uint4*>(p.k_vpt + ((size_t)t * p.Hkv + g) * 128 + 32 * wg);
            c0 = __ldg(src);
            c1 = __ldg(src + 1);
            ksb = __ldg(p.k_spt + ((size_t)t * p.Hkv + g) * 4 + wg);
          }
        } else {
          const uint8_t* krow = smem + oKpt + row * 128;
          c0 = *reinterpret_cast<const uint4*>(krow + (((2 * wg) ^ (row & 7)) << 4));
          c1 = *reinterpret_cast<const uint4*>(krow + (((2 * wg + 1) ^ (row & 7)) << 4));
          ksb = sfb(2)[16 * lane + 4 * quarter + wg];
        }
        const uint32_t codes[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t kd[16];
        dequant32_bf16(codes, ksb, kd);
        store_bf16_32(smem + oKd, row, wg, kd);
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(kd_full);
      }
      // rows past the document end get P = 0
      const float l2 = valid ? p.lse[(size_t)h * p.T + i] * kLog2e : INFINITY;
      const float dl = valid ? p.delta[(size_t)h * p.T + i] : 0.f;
      for (int v = 0; v < n; ++v, ++kt) {
        const bool diag = v == n - 1;
        // on the diagonal tile block `quarter` of this row is its own 32-key
        // block (per-token operands, second phase); later blocks are future keys
        const bool own = diag && wg == quarter;
        const bool future = diag && wg > quarter;
        uint32_t r[32];
        float ds[32];
        // ---- S -> P (in place)
        if (!take(s_full, s_free, s_cnt, tS, !own && !future, r)) { ok = false; break; }
        if (diag && !take(s_full, s_free, s_cnt, tS, own, r)) { ok = false; break; }
        if (future) {
#pragma unroll
          for (int c = 0; c < 32; ++c) ds[c] = 0.f;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float pp = fast_exp2(__uint_as_float(r[c]) * p.scale_log2 - l2);
            ds[c] = (!own || c <= lane) ? pp : 0.f;
          }
        }
        // ---- dP -> dS = P (dP - D)
        if (!take(dp_full, dp_free, dp_cnt, tDP, !own && !future, r)) { ok = false; break; }
        if (diag && !take(dp_full, dp_free, dp_cnt, tDP, own, r)) { ok = false; break; }
        if (!future) {
#pragma unroll
          for (int c = 0; c < 32; ++c) ds[c] = ds[c] * (__uint_as_float(r[c]) - dl);
        }
        uint32_t cw[8];
        const uint32_t sb = quant32(ds, p.rule, cw);
        uint32_t pd[16];
        if (own) {
          // the diagonal block leaves the FP8 operand (it goes through the bf16 MMA)
          dequant32_bf16(cw, sb, pd);
#pragma unroll
          for (int c = 0; c < 8; ++c) cw[c] = 0;
        }
        // dQ of the previous tile must have read the dS buffers
        if (kt > 0 && !warp_wait(dq_done, (kt - 1) & 1, wd, 80)) { ok = false; break; }
        store_codes32(sDS, row, 2 * wg, cw);
        sfDS[(row & 31) * 16 + (row >> 5) * 4 + wg] = (uint8_t)sb;
        if (diag) {
          if (!own) {
#pragma unroll
            for (int c = 0; c < 16; ++c) pd[c] = 0;
          }
          store_bf16_32(sDSd, row, wg, pd);
        }
        fence_proxy_async_smem();
        warp_arrive(ds_ready);
      }
      if (!ok) break;
      if (!warp_wait(acc_full, unit_i & 1, wd, 81)) break;
      tc_fence_after();
      {
        uint32_t t[32];
        tmem_ld32(lb + tDQ + 32 * wg, t);
        tmem_wait_ld(t);
        if (valid && 32 * wg < p.d)
          store_row32(p.out0, ((size_t)i * p.Hq + h) * p.d + 32 * wg, t, p.scale, p.grad_bf16, p.wide);
      }
      tc_fence_before();
      warp_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kMma) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
namespace kvk {
// warps 0-15: one thread per (key row, 32-query block): warpgroup wg on query
// block wg of every tile (one MX scale block of P~T and dS~T); warp 16: all
// loads (K/V; per query tile lse, D, Q^pt, dO^pt, dO^tb, Q^tb); warp 17: MMA
// issue.  18 warps leave 112 registers per thread (19 would leave 96).
constexpr int kThreads = 576, kLoadA = 16, kMma = 17, kComputeWarps = 16;
// per item: K^tb, K^pt, V^tb, V^pt codes; per query tile one buffer per
// operand (Q^pt, dO^pt, dO^tb, Q^tb codes), each released as soon as its last
// MMA has read it; P~T and dS~T codes; lse*log2e[128] and D[128] of the query
// tile in two buffers
constexpr int oKtb = 0, oKpt = oKtb + kCode, oVtb = oKpt + kCode, oVpt = oVtb + kCode;
constexpr int oQpt = oVpt + kCode, oDOpt = oQpt + kCode, oDOtb = oDOpt + kCode, oQtb = oDOtb + kCode;
constexpr int oP = oQtb + kCode, oDS = oP + kCode;
constexpr int oAux = oDS + kCode;
constexpr int oSf = oAux + 2 * 1024;
// scale blocks: 0 Ktb, 1 Kpt, 2 Vtb, 3 Vpt, 4 Qpt, 5 dOpt, 6 dOtb (channel rows), 7 Qtb (channel rows), 8 P, 9 dS,
// 10 (mixed path) Q's second NVFP4 block.  Mixed path: the NVFP4 K tile at oKtb with its two
// blocks in 0 and 1 (the per-token K is not loaded), the NVFP4 Q tile at oQpt
constexpr int kNumSf = 11;
constexpr int kNvTile = 128 * 64;
constexpr int oBars = oSf + kNumSf * kSfBlk;
// operand buffers, in the order the MMAs release them
constexpr int kQpt = 0, kDOpt = 1, kDOtb = 2, kQtb = 3;
// (bAuxFull, bDsFull: unused slots)
constexpr int bKvFull = 0, bKvEmpty = 1, bOpFull = 2, bOpEmpty = 6, bAuxFull = 10, bAuxEmpty = 12, bSFull = 14,
              bSFree = 15, bPFull = 16, bDsFull = 17, bAccFull = 18, bAccFree = 19, bFin = 20, bRing = 21,
              kNumBars = bRing + 2 * kUnitRing;  // the unit ring's full[], empty[] from bRing
constexpr int kSmem = oBars + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory exceeds the 227 KB a CTA may use");
// TMEM: one 128-column region that holds S^T and dP^T in turn (each read out
// into registers and released before the next), dV, dK, scale factors
constexpr uint32_t tSD = 0, tDV = 128, tDK = 256;
constexpr uint32_t tSfKtb = 384, tSfKpt = 388, tSfVtb = 392, tSfVpt = 396, tSfQpt = 400, tSfDOpt = 404, tSfP = 408,
                   tSfDS = 412, tSfDOtb = 416, tSfQtb = 420, tSfQ2 = 424;
constexpr uint32_t kSfCols[] = {tSfKtb, tSfKpt, tSfVtb, tSfVpt, tSfQpt, tSfDOpt, tSfP, tSfDS, tSfDOtb, tSfQtb, tSfQ2};
static_assert(sf_cols_ok(kSfCols, tDK + 128), "dK/dV kernel TMEM scale columns overlap");
}  // namespace kvk

// kNv: tm_ktb and tm_kpt map K's NVFP4 codes (only tm_ktb is read), tm_qpt Q's
template <bool kNv>
__global__ void __launch_bounds__(kvk::kThreads, 1)
    dkdv_mx_kernel(const __grid_constant__ CUtensorMap tm_ktb, const __grid_constant__ CUtensorMap tm_kpt,
                   const __grid_constant__ CUtensorMap tm_vtb, const __grid_constant__ CUtensorMap tm_vpt,
                   const __grid_constant__ CUtensorMap tm_qpt, const __grid_constant__ CUtensorMap tm_qtb,
                   const __grid_constant__ CUtensorMap tm_dopt, const __grid_constant__ CUtensorMap tm_dotb,
                   const MxParams p) {
  using namespace kvk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sf = smem + oSf;
  auto sfb = [&](int i) { return sf + i * kSfBlk; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* kv_full = bars + bKvFull;
  uint64_t* kv_empty = bars + bKvEmpty;
  uint64_t* op_full = bars + bOpFull;
  uint64_t* op_empty = bars + bOpEmpty;
  uint64_t* aux_empty = bars + bAuxEmpty;
  uint64_t* s_full = bars + bSFull;
  uint64_t* s_free = bars + bSFree;
  uint64_t* p_full = bars + bPFull;
  uint64_t* ds_full = bars + bDsFull;
  uint64_t* acc_full = bars + bAccFull;
  uint64_t* acc_free = bars + bAccFree;
  uint64_t* fin = bars + bFin;
  const UnitRing ring{reinterpret_cast<int*>(bars + kNumBars) + 4, bars + kNumBars - 2 * kUnitRing,
                      bars + kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 32);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(op_full + i, 32);  // lane 0's expect_tx arrive + 31 lanes after their scale stores
      mbar_init(op_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(aux_empty + i, kComputeWarps);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kComputeWarps);
    mbar_init(p_full, kComputeWarps);
    mbar_init(ds_full, kComputeWarps);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kComputeWarps);
    mbar_init(fin, 1);
    unit_ring_init(ring, 1 + kComputeWarps);  // the MMA thread and the compute warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMma) {
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
  auto decode = [&](const UnitInfo& un, int& doc, int& s, int& e, int& g, int& v, int& k0, int& nq) {
    doc = un.doc;
    v = un.tile;
    g = un.h;
    s = un.s;
    e = un.e;
    k0 = s + 128 * v;
    nq = (e - s + 127) / 128;
  };
  // one operand buffer of query tile t: wait until the MMAs of tile t - 1 released
  // it, store its scale block, then copy the codes
  // (mixed path, Q^pt buffer: Q's NVFP4 tile, its second scale block sfw2 in block 10)
  auto load_op = [&](int op, uint32_t t, const CUtensorMap* tm, int h, int q0, const uint4& sfw, int where,
                     const uint4* sfw2 = nullptr) {
    if (t > 0 && !warp_wait(op_empty + op, (t - 1) & 1, wd, where)) return false;
    reinterpret_cast<uint4*>(sfb(4 + op))[lane] = sfw;
    if (sfw2) reinterpret_cast<uint4*>(sfb(10))[lane] = *sfw2;
    fence_proxy_async_smem();
    const int off = op == kQpt ? oQpt : op == kDOpt ? oDOpt : op == kDOtb ? oDOtb : oQtb;
    if (lane == 0) {
      mbar_arrive_expect_tx(op_full + op, (kNv && op == kQpt) ? kNvTile : kCode);
      tma_load_3d(smem + off, tm, op_full + op, 0, h, q0);
    } else {
      mbar_arrive(op_full + op);
    }
    return true;
  };

  if (warp == kLoadA) {
    // ------------------------------------------------- K, V; Q^pt, dO^pt; lse, D
    uint32_t t = 0;
    int unit_i = 0;
    bool ok = true;
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_produce_warp(ring, us, p.cu, p.sched.next, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      int doc, s, e, g, v, k0, nq;
      decode(un, doc, s, e, g, v, k0, nq);
      if (unit_i > 0 && !warp_wait(kv_empty, (unit_i - 1) & 1, wd, 81)) break;
      if constexpr (kNv) {
        const uint2 w0 = nv_scale_words(p.k_nvs, k0 + lane, p.T, p.Hkv, g);
        const uint2 w1 = nv_scale_words(p.k_nvs, k0 + lane + 32, p.T, p.Hkv, g);
        const uint2 w2 = nv_scale_words(p.k_nvs, k0 + lane + 64, p.T, p.Hkv, g);
        const uint2 w3 = nv_scale_words(p.k_nvs, k0 + lane + 96, p.T, p.Hkv, g);
        reinterpret_cast<uint4*>(sfb(0))[lane] = make_uint4(w0.x, w1.x, w2.x, w3.x);
        reinterpret_cast<uint4*>(sfb(1))[lane] = make_uint4(w0.y, w1.y, w2.y, w3.y);
      } else {
        reinterpret_cast<uint4*>(sfb(0))[lane] = tb_rows(p.k_stb, s, e, doc, 4 * v, p.Hkv, g);
        reinterpret_cast<uint4*>(sfb(1))[lane] = pt_rows(p.k_spt, k0, lane, p.T, p.Hkv, g);
      }
      reinterpret_cast<uint4*>(sfb(2))[lane] = tb_rows(p.v_stb, s, e, doc, 4 * v, p.Hkv, g);
      reinterpret_cast<uint4*>(sfb(3))[lane] = pt_rows(p.v_spt, k0, lane, p.T, p.Hkv, g);
      fence_proxy_async_smem();
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, kNv ? kNvTile + 2 * kCode : 4 * kCode);
        tma_load_3d(smem + oKtb, &tm_ktb, kv_full, 0, g, k0);
        if (!kNv) tma_load_3d(smem + oKpt, &tm_kpt, kv_full, 0, g, k0);
        tma_load_3d(smem + oVtb, &tm_vtb, kv_full, 0, g, k0);
        tma_load_3d(smem + oVpt, &tm_vpt, kv_full, 0, g, k0);
      } else {
        mbar_arrive(kv_full);
      }
      for (int h = g * G; h < (g + 1) * G && ok; ++h) {
        for (int m = v; m < nq; ++m, ++t) {
          const int q0 = s + 128 * m;
          // all global reads of the tile first, so that their latencies overlap
          uint4 sq, sq2;
          if constexpr (kNv) {
            const uint2 w0 = nv_scale_words(p.q_nvs, q0 + lane, p.T, p.Hq, h);
            const uint2 w1 = nv_scale_words(p.q_nvs, q0 + lane + 32, p.T, p.Hq, h);
            const uint2 w2 = nv_scale_words(p.q_nvs, q0 + lane + 64, p.T, p.Hq, h);
            const uint2 w3 = nv_scale_words(p.q_nvs, q0 + lane + 96, p.T, p.Hq, h);
            sq = make_uint4(w0.x, w1.x, w2.x, w3.x);
            sq2 = make_uint4(w0.y, w1.y, w2.y, w3.y);
          } else {
            sq = pt_rows(p.q_spt, q0, lane, p.T, p.Hq, h);
          }
          const uint4 sdo = pt_rows(p.do_spt, q0, lane, p.T, p.Hq, h);
          float l4[4], d4[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int i = q0 + lane * 4 + r;
            const bool in = i < e;  // queries past the document end get P = 0 (-lse log2 e = -inf)
            l4[r] = in ? -p.lse[(size_t)h * p.T + i] * kLog2e : -INFINITY;
            d4[r] = in ? p.delta[(size_t)h * p.T + i] : 0.f;
          }
          const int ab = t & 1;
          if (t >= 2 && !warp_wait(aux_empty + ab, ((t >> 1) - 1) & 1, wd, 82)) { ok = false; break; }
          float* lse2 = reinterpret_cast<float*>(smem + oAux + ab * 1024);
          reinterpret_cast<float4*>(lse2)[lane] = make_float4(l4[0], l4[1], l4[2], l4[3]);
          reinterpret_cast<float4*>(lse2 + 128)[lane] = make_float4(d4[0], d4[1], d4[2], d4[3]);
          // no barrier of their own: each lane's arrival on Q^pt's barrier
          // below releases these stores, the MMA thread waits on that barrier
          // before it issues S^T of this tile, and the compute warps read them
          // only after they have seen that S^T complete
          if (!load_op(kQpt, t, &tm_qpt, h, q0, sq, 83, kNv ? &sq2 : nullptr)) { ok = false; break; }
          if (!load_op(kDOpt, t, &tm_dopt, h, q0, sdo, 84)) { ok = false; break; }
          // the query-side operands of dV and dK (token-block form)
          const uint4 sdotb = tb_channel_rows(p.do_stb, s, e, doc, 4 * m, p.Hq, h);
          const uint4 sqtb = tb_channel_rows(p.q_stb, s, e, doc, 4 * m, p.Hq, h);
          if (!load_op(kDOtb, t, &tm_dotb, h, q0, sdotb, 85)) { ok = false; break; }
          if (!load_op(kQtb, t, &tm_qtb, h, q0, sqtb, 86)) { ok = false; break; }
        }
      }
    }
    if (lane == 0) {
      if (unit_i > 0) drain_wait(kv_full, (unit_i - 1) & 1, p.timeout_ns);
      if (t > 0) {
        drain_wait(op_full + kQpt, (t - 1) & 1, p.timeout_ns);
        drain_wait(op_full + kDOpt, (t - 1) & 1, p.timeout_ns);
        drain_wait(op_full + kDOtb, (t - 1) & 1, p.timeout_ns);
        drain_wait(op_full + kQtb, (t - 1) & 1, p.timeout_ns);
      }
    }
  } else if (warp == kMma) {
    // ------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t aKtb = smem_u32(smem + oKtb), aKpt = smem_u32(smem + oKpt), aVtb = smem_u32(smem + oVtb),
                     aVpt = smem_u32(smem + oVpt), aQpt = smem_u32(smem + oQpt), aQtb = smem_u32(smem + oQtb),
                     aDOpt = smem_u32(smem + oDOpt), aDOtb = smem_u32(smem + oDOtb), aP = smem_u32(smem + oP),
                     aDS = smem_u32(smem + oDS), aSf = smem_u32(sf);
      uint32_t t = 0, s_uses = 0;
      int unit_i = 0;
      bool ok = true;
      auto mx_kk = [&](uint32_t dcol, uint32_t a, uint32_t b, uint32_t sfa, uint32_t sfbc, bool b_mn,
                       bool acc_first) {
        const uint64_t da = sdesc_sw128(a, 16, 1024), db = b_mn ? sdesc_sw128(b, 16384, 1024) : sdesc_sw128(b, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_mxf8_ss(tmem + dcol, da + ((kk * 32) >> 4), db + ((b_mn ? kk * 4096 : kk * 32) >> 4),
                      idesc_mxf8(128, 128, b_mn, kk, kk), (tmem + sfa) | ((uint32_t)kk << 30),
                      (tmem + sfbc) | ((uint32_t)kk << 30), (acc_first || kk > 0) ? 1u : 0u);
      };
      // the S/dP region: wait until the compute warps have read out its previous use
      auto region = [&]() {
        if (s_uses > 0 && !mbar_wait(s_free, (s_uses - 1) & 1, wd, 87)) return false;
        tc_fence_after();
        return true;
      };
      auto region_done = [&]() {
        tc_commit(s_full);
        ++s_uses;
      };
      auto wait_op = [&](int op, uint32_t tt, int where) {
        if (!mbar_wait(op_full + op, tt & 1, wd, where)) return false;
        tc_fence_after();
        return true;
      };
      // mixed path: S^T from the NVFP4 K (scale blocks at tSfKtb, tSfKpt) and Q (tSfQpt, tSfQ2)
      auto nv_st = [&]() {
        const uint64_t da = sdesc_sw64(aKtb), db = sdesc_sw64(aQpt);
        constexpr uint32_t idn = idesc_nvf4(128, 128);
        mma_nvf4_ss(tmem + tSD, da, db, idn, tmem + tSfKtb, tmem + tSfQpt, 0u);
        mma_nvf4_ss(tmem + tSD, da + 2, db + 2, idn, tmem + tSfKpt, tmem + tSfQ2, 1u);
      };
      // S^T of tile tt with token-block K (every key block of the tile)
      auto s_tb = [&](uint32_t tt) {
        if (!wait_op(kQpt, tt, 88)) return false;
        tmem_cp_sf(tmem + tSfQpt, aSf + 4 * kSfBlk);
        if (kNv) tmem_cp_sf(tmem + tSfQ2, aSf + 10 * kSfBlk);
        if (!region()) return false;
        if (kNv)
          nv_st();
        else
          mx_kk(tSD, aKtb, aQpt, tSfKtb, tSfQpt, false, false);
        region_done();
        return true;
      };
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
          const int w = un.w;
        if (w < 0 || w >= n_units) break;
        int doc, s, e, g, v, k0, nq;
        decode(un, doc, s, e, g, v, k0, nq);
        if (!mbar_wait(kv_full, unit_i & 1, wd, 89)) break;
        if (unit_i > 0 && !mbar_wait(acc_free, (unit_i - 1) & 1, wd, 90)) break;
        tc_fence_after();
        tmem_cp_sf(tmem + tSfKtb, aSf + 0 * kSfBlk);
        tmem_cp_sf(tmem + tSfKpt, aSf + 1 * kSfBlk);
        tmem_cp_sf(tmem + tSfVtb, aSf + 2 * kSfBlk);
        tmem_cp_sf(tmem + tSfVpt, aSf + 3 * kSfBlk);
        const int nt = nq - v, R = G * nt;
        bool ahead = false;  // S^T (token-block K) of tile t already issued
        for (int r = 0; r < R; ++r, ++t) {
          const bool diag = (r % nt) == 0;  // first query tile of each head: the diagonal tile
          const bool last = r == R - 1;
          if (!ahead && !s_tb(t)) { ok = false; break; }
          if (diag) {
            // diagonal tile: S^T again with the per-token K; the compute warps
            // take its diagonal 32x32 blocks
            // (mixed path: the same NVFP4 product again)
            if (!region()) { ok = false; break; }
            if (kNv)
              nv_st();
            else
              mx_kk(tSD, aKpt, aQpt, tSfKpt, tSfQpt, false, false);
            region_done();
          }
          tc_commit(op_empty + kQpt);
          // dP^T (token-block V), on the diagonal tile then the per-token V
          if (!wait_op(kDOpt, t, 91)) { ok = false; break; }
          tmem_cp_sf(tmem + tSfDOpt, aSf + 5 * kSfBlk);
          if (!region()) { ok = false; break; }
          mx_kk(tSD, aVtb, aDOpt, tSfVtb, tSfDOpt, false, false);
          region_done();
          if (diag) {
            if (!region()) { ok = false; break; }
            mx_kk(tSD, aVpt, aDOpt, tSfVpt, tSfDOpt, false, false);
            region_done();
          }
          tc_commit(op_empty + kDOpt);
          if (last) tc_commit(kv_empty);  // the item's last read of K and V has been issued
          // dV += P~T dO~tb
          if (!mbar_wait(p_full, t & 1, wd, 92)) { ok = false; break; }
          if (!wait_op(kDOtb, t, 93)) { ok = false; break; }
          tmem_cp_sf(tmem + tSfP, aSf + 8 * kSfBlk);
          tmem_cp_sf(tmem + tSfDOtb, aSf + 6 * kSfBlk);
          mx_kk(tDV, aP, aDOtb, tSfP, tSfDOtb, true, r > 0);
          tc_commit(op_empty + kDOtb);
          // the next tile's S^T goes ahead of dK, so that it is ready when the
          // compute warps finish dS~ of this tile
          ahead = false;
          if (!last) {
            if (!s_tb(t + 1)) { ok = false; break; }
            ahead = true;
          }
          // dK += dS~T Q~tb
          if (!mbar_wait(ds_full, t & 1, wd, 94)) { ok = false; break; }
          if (!wait_op(kQtb, t, 95)) { ok = false; break; }
          tmem_cp_sf(tmem + tSfDS, aSf + 9 * kSfBlk);
          tmem_cp_sf(tmem + tSfQtb, aSf + 7 * kSfBlk);
          mx_kk(tDK, aDS, aQtb, tSfDS, tSfQtb, true, r > 0);
          tc_commit(op_empty + kQtb);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp < kComputeWarps) {
    // ------------------------------------------------- P~T, dS~T
    // one thread per (key row, query block wg)
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lb = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sP = smem + oP;
    uint8_t* sDS = smem + oDS;
    uint8_t* sfP = sfb(8);
    uint8_t* sfDS = sfb(9);
    uint32_t s_cnt = 0, t = 0;
    int unit_i = 0;
    bool ok = true;
    // one use of the S/dP region: wait for it, read this thread's block if
    // `load`, release it
    auto take = [&](bool load, uint32_t (&r)[32]) {
      if (!warp_wait(s_full, s_cnt & 1, wd, 96)) return false;
      ++s_cnt;
      tc_fence_after();
      if (load) {
        tmem_ld32(lb + tSD + 32 * wg, r);
        tmem_wait_ld(r);
      }
      tc_fence_before();
      warp_arrive(s_free);
      return true;
    };
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      int doc, s, e, g, v, k0, nq;
      decode(un, doc, s, e, g, v, k0, nq);
      const int j = k0 + row;
      for (int h = g * G; h < (g + 1) * G && ok; ++h) {
        for (int m = v; m < nq; ++m, ++t) {
          const bool diag = m == v;
          // on the diagonal tile query block `quarter` is this key row's own
          // 32-query block (per-token operands, second phase); earlier query
          // blocks precede the key (P = 0)
          const bool own = diag && wg == quarter;
          const bool past = diag && wg < quarter;
          const int ab = t & 1;
          // -lse log2 e and D of this block's 32 queries (identical across the
          // warp), read after S^T of this tile has been seen complete
          const float4* nl4 = reinterpret_cast<const float4*>(smem + oAux + ab * 1024) + 8 * wg;
          const float4* dl4 = nl4 + 32;
          uint32_t r[32];
          uint64_t pr2[16];  // P of this thread's 32 queries, in pairs (kept for dS)
          // ---- S^T -> P (kept in registers), P~T into shared memory
          if (!take(!own && !past, r)) { ok = false; break; }
          if (diag && !take(own, r)) { ok = false; break; }
          if (past) {
#pragma unroll
            for (int i = 0; i < 16; ++i) pr2[i] = 0ull;
          } else {
            // P = 2^(S scale log2 e - lse log2 e): one packed FMA per pair
            const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 n = nl4[q];
              float a0, a1, a2, a3;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), sl2,
                               f2_pack(n.x, n.y)), a0, a1);
              f2_unpack(f2_fma(f2_pack(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])), sl2,
                               f2_pack(n.z, n.w)), a2, a3);
              pr2[2 * q] = f2_pack(fast_exp2(a0), fast_exp2(a1));
              pr2[2 * q + 1] = f2_pack(fast_exp2(a2), fast_exp2(a3));
            }
            if (own) {
              // on the own block query column c is visible iff it is >= the key row
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float lo, hi;
                f2_unpack(pr2[i], lo, hi);
                pr2[i] = f2_pack(2 * i >= lane ? lo : 0.f, 2 * i + 1 >= lane ? hi : 0.f);
              }
            }
          }
          // P~T's buffer and scale block are free: this thread has seen S^T of
          // this tile complete, and the MMA thread issued that S^T after the
          // previous tile's dV MMA and scale copy (a commit tracks every earlier
          // tcgen05 operation of its thread)
          {
            uint32_t cw[8];
            const uint32_t sb = mx_quant32_pairs<true>(pr2, p.rule, cw);
            store_codes32(sP, row, 2 * wg, cw);
            sfP[(row & 31) * 16 + (row >> 5) * 4 + wg] = (uint8_t)sb;
          }
          fence_proxy_async_smem();
          warp_arrive(p_full);
          // ---- dP^T -> dS~T into shared memory
          if (!take(!own && !past, r)) { ok = false; break; }
          if (diag && !take(own, r)) { ok = false; break; }
          // dS~T's buffer is free likewise: dP^T of this tile was issued after
          // the previous tile's dK MMA
          {
            // dS = P (dP - D), packed, in place of P (P is not needed after this)
            if (!past) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 dd = dl4[q];
                pr2[2 * q] = f2_mul(pr2[2 * q], f2_sub(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])),
                                                      f2_pack(dd.x, dd.y)));
                pr2[2 * q + 1] = f2_mul(pr2[2 * q + 1], f2_sub(f2_pack(__uint_as_float(r[4 * q + 2]),
                                                                      __uint_as_float(r[4 * q + 3])),
                                                              f2_pack(dd.z, dd.w)));
              }
            }
            uint32_t cw[8];
            const uint32_t sb = mx_quant32_pairs<false>(pr2, p.rule, cw);
            store_codes32(sDS, row, 2 * wg, cw);
            sfDS[(row & 31) * 16 + (row >> 5) * 4 + wg] = (uint8_t)sb;
          }
          fence_proxy_async_smem();
          warp_arrive(ds_full);
          warp_arrive(aux_empty + ab);
        }
      }
      if (!ok) break;
      // epilogue: warpgroups 0, 1 write halves of dV, warpgroups 2, 3 halves of dK * scale
      if (!warp_wait(acc_full, unit_i & 1, wd, 100)) break;
      tc_fence_after();
      const bool valid = j < e;
      const bool is_k = wg >= 2;
      const int c0 = (wg & 1) * 64;
      const uint32_t acc = lb + (is_k ? tDK : tDV) + c0;
      void* out = is_k ? p.out0 : p.out1;
      const float mul = is_k ? p.scale : 1.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t tt[32];
        tmem_ld32(acc + 32 * c, tt);
        tmem_wait_ld(tt);
        if (valid && c0 + 32 * c < p.d)
          store_row32(out, ((size_t)j * p.Hkv + g) * p.d + c0 + 32 * c, tt, mul, p.grad_bf16, p.wide);
      }
      tc_fence_before();
      warp_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kMma) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_bwd_mxfp8(const BwdMxArgs& a, cudaStream_t stream) {
  // 1. D = rowsum(dO * (o + residual)) and dO's two MX forms, in one read of dO
  a.marks.at(2, stream);
  {
    QuantJob job{static_cast<const __nv_bfloat16*>(a.dout), a.Hq, const_cast<uint8_t*>(a.do_vtb),
                 const_cast<uint8_t*>(a.do_stb), const_cast<uint8_t*>(a.do_vpt), const_cast<uint8_t*>(a.do_spt),
                 nullptr, true};
    DeltaArgs da;
    da.o = static_cast<const __nv_bfloat16*>(a.o);
    da.o_resid = static_cast<const __nv_bfloat16*>(a.o_resid);
    da.delta = a.delta;
    da.T = a.T;
    cudaError_t e = launch_quantize_with_delta(job, a.T, a.d, a.cu, a.n_docs, a.rule, da, stream);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tqpt, tqtb, tktb, tkpt, tvtb, tvpt, tdopt, tdotb, tqnv, tknv;
  if (!make_tmap_codes(&tqtb, a.q_vtb, a.T, a.Hq) || !make_tmap_codes(&tktb, a.k_vtb, a.T, a.Hkv) ||
      !make_tmap_codes(&tkpt, a.k_vpt, a.T, a.Hkv) || !make_tmap_codes(&tvtb, a.v_vtb, a.T, a.Hkv) ||
      !make_tmap_codes(&tvpt, a.v_vpt, a.T, a.Hkv) || !make_tmap_codes(&tdopt, a.do_vpt, a.T, a.Hq) ||
      !make_tmap_codes(&tdotb, a.do_vtb, a.T, a.Hq))
    return cudaErrorInvalidValue;
  if (a.nv) {
    // the scores' operands: NVFP4 Q and K (Q's per-token MXFP8 form is not kept)
    if (!make_tmap_nv(&tqnv, a.q_nvv, a.T, a.Hq) || !make_tmap_nv(&tknv, a.k_nvv, a.T, a.Hkv))
      return cudaErrorInvalidValue;
    tqpt = tqnv;
  } else {
    if (!make_tmap_codes(&tqpt, a.q_vpt, a.T, a.Hq)) return cudaErrorInvalidValue;
    tknv = tkpt;  // not read
  }
  MxParams p;
  p.cu = a.cu;
  p.lse = a.lse;
  p.delta = a.delta;
  p.q_stb = a.q_stb; p.q_spt = a.q_spt;
  p.k_stb = a.k_stb; p.k_spt = a.k_spt;
  p.v_stb = a.v_stb; p.v_spt = a.v_spt;
  p.do_stb = a.do_stb; p.do_spt = a.do_spt;
  p.q_nvs = a.q_nvs; p.k_nvs = a.k_nvs; p.k_vpt = a.k_vpt;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.d;
  p.scale = a.scale;
  // mixed path: the scores' MMAs leave out the decode scales of Q and K
  p.scale_log2 = a.scale * kLog2e * (a.nv ? a.nv_g_q * a.nv_g_k : 1.f);
  p.grad_bf16 = a.grad_bf16;
  p.rule = a.rule;
  // 2. dK, dV
  a.marks.at(3, stream);
  {
    const auto kern = a.nv ? dkdv_mx_kernel<true> : dkdv_mx_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kvk::kSmem);
    if (e != cudaSuccess) return e;
    MxParams pk = p;
    pk.sched = sched_view(a.sched_kv);
    pk.cta_times = a.cta_times[0];
    pk.out0 = a.dk;
    pk.out1 = a.dv;
    pk.wide = aligned32(a.dk) && aligned32(a.dv);
    const long long max_units = (long long)a.sched_kv.max_items * a.Hkv;
    const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
    if (a.nv)
      kern<<<grid, kvk::kThreads, kvk::kSmem, stream>>>(tknv, tknv, tvtb, tvpt, tqpt, tqtb, tdopt, tdotb, pk);
    else
      kern<<<grid, kvk::kThreads, kvk::kSmem, stream>>>(tktb, tkpt, tvtb, tvpt, tqpt, tqtb, tdopt, tdotb, pk);
    note_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 3. dQ
  a.marks.at(4, stream);
  {
    const auto kern = a.nv ? dq_mx_kernel<true> : dq_mx_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::kSmem);
    if (e != cudaSuccess) return e;
    MxParams pq = p;
    pq.sched = sched_view(a.sched_q);
    pq.cta_times = a.cta_times[1];
    pq.out0 = a.dq;
    pq.wide = aligned32(a.dq);
    pq.out1 = nullptr;
    const long long max_units = (long long)a.sched_q.max_items * a.Hq;
    const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
    kern<<<grid, dqk::kThreads, dqk::kSmem, stream>>>(tqpt, tdopt, tktb, tvtb, tkpt, tvpt, tknv, pq);
    note_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  a.marks.at(5, stream);
  return cudaSuccess;
}

}  // namespace fapk
